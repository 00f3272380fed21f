"""The prefill kernel's FMA-pipe 2^x: its constants, evaluated the way the kernel does
in fp32 (rounding shift, remainder, Horner, exponent add), stay within the stated
relative error over the softmax's whole input range, far below bf16's half ulp."""
import pathlib
import re

import numpy as np

SRC = pathlib.Path(__file__).resolve().parents[1] / "cross_layer_kv_shared_b200" / "csrc" / "prefill_sm100.cu"


def constants():
    text = SRC.read_text()
    c = {k: np.float32(float(v)) for k, v in re.findall(r"constexpr float (EXP2_C\d) = ([0-9.eE+-]+)f;", text)}
    assert sorted(c) == ["EXP2_C0", "EXP2_C1", "EXP2_C2", "EXP2_C3"]
    return c


def exp2_fma(x, c):
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    shift = f32(12582912.0)
    t = (x + shift).astype(f32)
    f = (x - (t - shift).astype(f32)).astype(f32)
    p = f32(c["EXP2_C3"])
    for k in ("EXP2_C2", "EXP2_C1", "EXP2_C0"):
        p = (p * f + c[k]).astype(f32)        # fmaf rounds once; two roundings here only add error
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(f32)


def test_relative_error_over_softmax_range():
    c = constants()
    x = np.linspace(-124.0, 8.0, 2_000_001).astype(np.float32)
    got = exp2_fma(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1.0e-4, rel.max()
    assert rel.max() < 2.0 ** -9 / 20          # bf16 half ulp is 2^-9


def test_integers_and_clamp():
    c = constants()
    x = np.arange(-125, 9, dtype=np.float32)
    got = exp2_fma(x, c).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1) < 1e-4)
    low = exp2_fma(np.array([-126.0, -300.0, -np.inf], dtype=np.float32), c)
    assert np.all(np.isfinite(low)) and np.all(low > 0) and np.all(low < 2.0 ** -124)
