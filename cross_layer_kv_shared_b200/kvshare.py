"""ctypes binding of libkvshare (include/kvshare.h): argument marshalling only.

Every function keeps the C name. Tensors are torch tensors on the CUDA device
(torch is used for device memory and streams only); every step of the
computation runs in the library's kernels. A missing library raises at import:
there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvshare.so")

KVS_OK, KVS_EINVAL, KVS_EUNSUPPORTED, KVS_ENOMEM, KVS_ECUDA, KVS_ETIMEOUT = range(6)
KVS_F32, KVS_BF16 = 0, 1
KVS_SRC_SINGLE, KVS_SRC_MIX, KVS_SRC_LOWRANK = 0, 1, 2


class kvshare_config(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int), ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("dtype", ctypes.c_int), ("softmax_scale", ctypes.c_float),
                ("basis_rank", ctypes.c_int), ("max_resid_rank", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("max_context", ctypes.c_int)]


class kvshare_layer(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("src0", ctypes.c_int), ("src1", ctypes.c_int)]


class kvshare_cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("slots", ctypes.c_int),
                ("coef_k", ctypes.c_void_p), ("coef_v", ctypes.c_void_p),
                ("basis_k", ctypes.c_void_p), ("basis_v", ctypes.c_void_p),
                ("u_k", ctypes.c_void_p), ("u_v", ctypes.c_void_p),
                ("s_k", ctypes.c_void_p), ("s_v", ctypes.c_void_p),
                ("r_k", ctypes.c_void_p), ("r_v", ctypes.c_void_p),
                ("rank", ctypes.c_void_p), ("pairs", ctypes.c_int),
                ("batch", ctypes.c_int), ("context", ctypes.c_int),
                ("lengths", ctypes.c_void_p)]


class KVShareError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {kvshare_status_string(status)} (status {status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m cross_layer_kv_shared_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, V = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
    sig = {
        "kvshare_create": ([ctypes.POINTER(kvshare_config), ctypes.POINTER(ctypes.c_void_p)], I),
        "kvshare_destroy": ([P], I),
        "kvshare_set_map": ([P, ctypes.POINTER(kvshare_layer), P], I),
        "kvshare_decode": ([P, ctypes.POINTER(kvshare_cache), P, P, P, I, I, V], I),
        "kvshare_decode_host": ([P, ctypes.POINTER(kvshare_cache), P, P, P, I, I, V], I),
        "kvshare_decode_stats": ([P, ctypes.POINTER(kvshare_cache), P, P, P, P, P, P, P, I, I, V], I),
        "kvshare_prefill": ([P, ctypes.POINTER(kvshare_cache), P, P, P, I, I, I, V], I),
        "kvshare_pack_residual": ([P, P, P, P, P, P, P, P, P, I, I, V], I),
        "kvshare_append_lowrank": ([P, ctypes.POINTER(kvshare_cache), P, P, P, P, V], I),
        "kvshare_sync_status": ([P, V], I),
        "kvshare_set_splits": ([P, I], I),
        "kvshare_set_kv_overlap": ([P, I], I),
        "kvshare_set_layer_order": ([P, P], I),
        "kvshare_debug_stall_next": ([P, I], I),
        "kvshare_debug_set_grid": ([P, I], I),
        "kvshare_launch_count": ([P], ctypes.c_uint64),
        "kvshare_status_string": ([I], ctypes.c_char_p),
        "kvshare_decode_layer_noalloc": ([P, P, P, P, P, P, I, I, I, I, I, I, I, I, V], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _load()


def kvshare_status_string(status: int) -> str:
    return _lib.kvshare_status_string(int(status)).decode()


def _check(status: int, where: str) -> int:
    if status != KVS_OK:
        raise KVShareError(status, where)
    return status


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return int(t.data_ptr()) if hasattr(t, "data_ptr") else int(t)


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    return int(getattr(stream, "cuda_stream", stream))


def kvshare_create(num_layers: int, num_q_heads: int, num_kv_heads: int, head_dim: int, dtype: int,
                   max_batch: int, max_context: int, softmax_scale: float = 0.0, basis_rank: int = 32,
                   max_resid_rank: int = 16, check: bool = True):
    """Returns (status, handle); raises KVShareError on failure when ``check``."""
    cfg = kvshare_config(num_layers, num_q_heads, num_kv_heads, head_dim, dtype, softmax_scale, basis_rank,
                         max_resid_rank, max_batch, max_context)
    h = ctypes.c_void_p()
    st = _lib.kvshare_create(ctypes.byref(cfg), ctypes.byref(h))
    if check:
        _check(st, "kvshare_create")
    return st, h


def kvshare_destroy(h) -> int:
    return _lib.kvshare_destroy(h)


def kvshare_set_map(h, layer_map: Sequence, w=None, check: bool = True) -> int:
    """layer_map: (kind, src0, src1) per layer; w: host float32 array [L][Hkv] or None."""
    arr = (kvshare_layer * len(layer_map))(*[kvshare_layer(int(k), int(a), int(b)) for k, a, b in layer_map])
    wp = None
    keep = None
    if w is not None:
        import numpy as np
        keep = np.ascontiguousarray(np.asarray(w, dtype=np.float32))
        wp = keep.ctypes.data
    st = _lib.kvshare_set_map(h, arr, wp)
    if check:
        _check(st, "kvshare_set_map")
    return st


@dataclass
class Cache:
    """Device tensors of a shared cache (fields as in kvshare_cache)."""
    batch: int
    context: int
    k: object = None
    v: object = None
    slots: int = 0
    coef_k: object = None
    coef_v: object = None
    basis_k: object = None
    basis_v: object = None
    u_k: object = None
    u_v: object = None
    s_k: object = None
    s_v: object = None
    r_k: object = None
    r_v: object = None
    rank: object = None
    pairs: int = 0
    lengths: object = None      # [batch] int32 device tensor of per-sequence token counts

    def as_c(self) -> kvshare_cache:
        p = lambda t: _ptr(t) or None  # noqa: E731
        return kvshare_cache(p(self.k), p(self.v), self.slots, p(self.coef_k), p(self.coef_v), p(self.basis_k),
                             p(self.basis_v), p(self.u_k), p(self.u_v), p(self.s_k), p(self.s_v), p(self.r_k),
                             p(self.r_v), p(self.rank), self.pairs, self.batch, self.context, p(self.lengths))


def kvshare_decode(h, cache: Cache, q, out, lse=None, l0: int = 0, l1: int = None, stream=None,
                   check: bool = True) -> int:
    c = cache.as_c()
    st = _lib.kvshare_decode(h, ctypes.byref(c), _ptr(q), _ptr(out), _ptr(lse), int(l0),
                             int(l1 if l1 is not None else q.shape[0]), _stream(stream))
    if check:
        _check(st, "kvshare_decode")
    return st


def kvshare_decode_stats(h, cache: Cache, q, out, lse, mass=None, score=None, entropy=None, peak=None,
                         l0: int = 0, l1: int = None, stream=None, check: bool = True) -> int:
    c = cache.as_c()
    st = _lib.kvshare_decode_stats(h, ctypes.byref(c), _ptr(q), _ptr(out), _ptr(lse), _ptr(mass), _ptr(score),
                                   _ptr(entropy), _ptr(peak), int(l0), int(l1 if l1 is not None else q.shape[0]),
                                   _stream(stream))
    if check:
        _check(st, "kvshare_decode_stats")
    return st


def kvshare_decode_host(h, cache: Cache, q_host, out_host, lse_host=None, l0: int = 0, l1: int = None,
                        stream=None, check: bool = True) -> int:
    c = cache.as_c()
    st = _lib.kvshare_decode_host(h, ctypes.byref(c), _ptr(q_host), _ptr(out_host), _ptr(lse_host), int(l0),
                                  int(l1 if l1 is not None else q_host.shape[0]), _stream(stream))
    if check:
        _check(st, "kvshare_decode_host")
    return st


def kvshare_prefill(h, cache: Cache, q, out, lse=None, l0: int = 0, l1: int = None, seqlen: int = None,
                    stream=None, check: bool = True) -> int:
    c = cache.as_c()
    st = _lib.kvshare_prefill(h, ctypes.byref(c), _ptr(q), _ptr(out), _ptr(lse), int(l0),
                              int(l1 if l1 is not None else q.shape[0]),
                              int(seqlen if seqlen is not None else q.shape[3]), _stream(stream))
    if check:
        _check(st, "kvshare_prefill")
    return st


def kvshare_pack_residual(h, score, u_k, u_v, rank, u_k8, u_v8, s_k, s_v, batch: int, context: int,
                          stream=None, check: bool = True) -> int:
    st = _lib.kvshare_pack_residual(h, _ptr(score), _ptr(u_k), _ptr(u_v), _ptr(rank), _ptr(u_k8), _ptr(u_v8),
                                    _ptr(s_k), _ptr(s_v), int(batch), int(context), _stream(stream))
    if check:
        _check(st, "kvshare_pack_residual")
    return st


def kvshare_append_lowrank(h, cache: Cache, k_new, v_new, score, pos, stream=None, check: bool = True) -> int:
    c = cache.as_c()
    st = _lib.kvshare_append_lowrank(h, ctypes.byref(c), _ptr(k_new), _ptr(v_new), _ptr(score), _ptr(pos),
                                     _stream(stream))
    if check:
        _check(st, "kvshare_append_lowrank")
    return st


def kvshare_sync_status(h, stream=None) -> int:
    return _lib.kvshare_sync_status(h, _stream(stream))


def kvshare_set_splits(h, splits: int) -> int:
    return _check(_lib.kvshare_set_splits(h, int(splits)), "kvshare_set_splits")


def kvshare_set_kv_overlap(h, on: bool = True) -> int:
    return _check(_lib.kvshare_set_kv_overlap(h, 1 if on else 0), "kvshare_set_kv_overlap")


def kvshare_set_layer_order(h, order=None, check: bool = True) -> int:
    """order: sequence of num_layers distinct layer indices, or None for model order."""
    keep = None
    if order is not None:
        keep = (ctypes.c_int * len(order))(*[int(x) for x in order])
    st = _lib.kvshare_set_layer_order(h, keep)
    if check:
        _check(st, "kvshare_set_layer_order")
    return st


def kvshare_debug_set_grid(h, ctas: int) -> int:
    return _check(_lib.kvshare_debug_set_grid(h, int(ctas)), "kvshare_debug_set_grid")


def kvshare_debug_stall_next(h, on: bool = True) -> int:
    return _check(_lib.kvshare_debug_stall_next(h, 1 if on else 0), "kvshare_debug_stall_next")


def kvshare_launch_count(h) -> int:
    return int(_lib.kvshare_launch_count(h))


def kvshare_decode_layer_noalloc(q, k, v, w, out, lse, batch: int, num_q_heads: int, num_kv_heads: int,
                                 head_dim: int, context: int, slots: int, src0: int, src1: int = -1,
                                 stream=None, check: bool = True) -> int:
    """One bf16 decode layer whose scratch lives in the library's fixed device array (no allocation)."""
    st = _lib.kvshare_decode_layer_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(w), _ptr(out), _ptr(lse), int(batch),
                                           int(num_q_heads), int(num_kv_heads), int(head_dim), int(context),
                                           int(slots), int(src0), int(src1), _stream(stream))
    if check:
        _check(st, "kvshare_decode_layer_noalloc")
    return st
