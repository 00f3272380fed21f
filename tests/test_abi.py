"""The C ABI: the libraries load without a GPU and export every symbol the headers declare."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBS = {
    "kvshare.h": os.path.join(ROOT, "cross_layer_kv_shared_b200", "libkvshare.so"),
    "kvsynth.h": os.path.join(ROOT, "synth", "libkvsynth.so"),
}


@pytest.fixture(scope="module", autouse=True)
def built():
    import __graft_entry__
    __graft_entry__.build()


def declared(header):
    with open(os.path.join(ROOT, "include", header)) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(kv[a-z0-9_]+)\s*\(", text, re.M)))


def exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib], capture_output=True, text=True, check=True).stdout
    return {line.split()[-1] for line in out.splitlines() if " T " in line}


@pytest.mark.parametrize("header", sorted(LIBS))
def test_every_declared_symbol_is_exported(header):
    names = declared(header)
    assert len(names) >= 2
    missing = set(names) - exported(LIBS[header])
    assert not missing, missing


def test_kvshare_entry_points_present():
    names = declared("kvshare.h")
    for n in ("kvshare_create", "kvshare_set_map", "kvshare_decode", "kvshare_prefill", "kvshare_destroy",
              "kvshare_pack_residual", "kvshare_sync_status", "kvshare_status_string", "kvshare_decode_host"):
        assert n in names


def test_libraries_load_and_status_strings_without_gpu():
    from cross_layer_kv_shared_b200 import kvshare as K
    assert K.kvshare_status_string(K.KVS_OK) == "ok"
    assert K.kvshare_status_string(K.KVS_ETIMEOUT) == "device wait timed out"
    assert K.kvshare_status_string(99) == "unknown status"
    ctypes.CDLL(LIBS["kvsynth.h"])


def test_null_arguments_are_rejected_without_touching_the_gpu():
    from cross_layer_kv_shared_b200 import kvshare as K
    lib = K._lib
    assert lib.kvshare_create(None, None) == K.KVS_EINVAL
    h = ctypes.c_void_p()
    assert lib.kvshare_create(None, ctypes.byref(h)) == K.KVS_EINVAL and not h.value
    assert lib.kvshare_destroy(None) == K.KVS_OK
    assert lib.kvshare_set_map(None, None, None) == K.KVS_EINVAL
    assert lib.kvshare_decode(None, None, None, None, None, 0, 0, None) == K.KVS_EINVAL
    assert lib.kvshare_sync_status(None, None) == K.KVS_EINVAL
    assert lib.kvshare_launch_count(None) == 0
    bad = K.kvshare_config(4, 6, 4, 64, K.KVS_BF16, 0.0, 32, 16, 1, 128)      # Hq % Hkv != 0
    assert lib.kvshare_create(ctypes.byref(bad), ctypes.byref(h)) == K.KVS_EINVAL
    bad = K.kvshare_config(4, 8, 4, 96, K.KVS_BF16, 0.0, 32, 16, 1, 128)      # head_dim 96
    assert lib.kvshare_create(ctypes.byref(bad), ctypes.byref(h)) == K.KVS_EUNSUPPORTED
    bad = K.kvshare_config(4, 64, 2, 64, K.KVS_BF16, 0.0, 32, 16, 1, 128)     # group of 32 > 16
    assert lib.kvshare_create(ctypes.byref(bad), ctypes.byref(h)) == K.KVS_EUNSUPPORTED


def test_unsupported_low_rank_and_scale_settings_are_rejected_without_touching_the_gpu():
    from cross_layer_kv_shared_b200 import kvshare as K
    lib = K._lib
    h = ctypes.c_void_p()

    def create(**kw):
        f = dict(L=4, Hq=8, Hkv=4, d=64, dt=K.KVS_BF16, scale=0.0, rb=32, rm=16, B=1, T=128)
        f.update(kw)
        c = K.kvshare_config(f["L"], f["Hq"], f["Hkv"], f["d"], f["dt"], f["scale"], f["rb"], f["rm"], f["B"], f["T"])
        return lib.kvshare_create(ctypes.byref(c), ctypes.byref(h))

    assert create(rb=48) == K.KVS_EUNSUPPORTED             # basis rank: 32 or head_dim only
    assert create(d=64, rb=128) == K.KVS_EUNSUPPORTED      # full rank means Rb = d
    assert create(rm=8) == K.KVS_EUNSUPPORTED              # residual rank fixed at 16
    assert create(scale=-1.0) == K.KVS_EINVAL
    assert create(scale=float("nan")) == K.KVS_EINVAL
    assert create(scale=float("inf")) == K.KVS_EINVAL
    assert create(dt=7) == K.KVS_EINVAL
    assert create(B=0) == K.KVS_EINVAL and create(T=0) == K.KVS_EINVAL and create(L=0) == K.KVS_EINVAL
    assert not h.value


def test_noalloc_shape_and_source_checks_run_before_any_cuda_call():
    from cross_layer_kv_shared_b200 import kvshare as K
    f = K._lib.kvshare_decode_layer_noalloc

    def call(B=2, Hq=8, Hkv=2, d=64, T=64, slots=2, s0=0, s1=-1):
        return f(None, None, None, None, None, None, B, Hq, Hkv, d, T, slots, s0, s1, None)

    assert call(B=0) == K.KVS_EINVAL and call(T=0) == K.KVS_EINVAL and call(slots=0) == K.KVS_EINVAL
    assert call(Hq=6, Hkv=4) == K.KVS_EINVAL                 # Hq % Hkv != 0
    assert call(d=96) == K.KVS_EUNSUPPORTED
    assert call(Hq=64, Hkv=2) == K.KVS_EUNSUPPORTED          # group of 32 > 16
    assert call(s0=2) == K.KVS_EINVAL and call(s0=-1) == K.KVS_EINVAL
    assert call(s1=2) == K.KVS_EINVAL and call(s1=0) == K.KVS_EINVAL   # mix source out of range / same as src0
    assert call(B=2049, Hkv=2, Hq=2) == K.KVS_EINVAL          # 4098 units > 4096
    assert call() == K.KVS_EINVAL                             # valid shape, but null (non-device) pointers
