"""The GPU generator reproduces the numpy generator's bits."""
import numpy as np
import pytest

from synth import philox
import synth.gpu as sgpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("offset,count", [(0, 1), (0, 4099), (3, 1000), (6, 7), ((1 << 33) + 1, 513)])
def test_normal_bits_match(offset, count):
    import torch
    for dt, tdt in (("f32", torch.float32), ("bf16", torch.bfloat16)):
        t = torch.empty(count, dtype=tdt, device="cuda")
        sgpu.fill_normal(t, 20261205, 9, 0.25, offset=offset)
        z = (philox.normal_f64(count, offset, 20261205, 9) * 0.25).astype(np.float32)
        want = z if dt == "f32" else philox.f32_bits_to_bf16_bits(z)
        got = t.cpu().numpy() if dt == "f32" else t.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got.view(np.uint32 if dt == "f32" else np.uint16),
                              want.view(np.uint32 if dt == "f32" else np.uint16))


@pytest.mark.parametrize("offset,count", [(0, 5), (1, 100003)])
def test_uniform_bits_match(offset, count):
    import torch
    t = torch.empty(count, dtype=torch.float32, device="cuda")
    sgpu.fill_uniform(t, 7, 13, offset=offset)
    w = philox.raw_words(count, offset, 7, 13)
    want = ((w >> np.uint64(8)).astype(np.float64) * 2.0 ** -24).astype(np.float32)
    assert np.array_equal(t.cpu().numpy(), want)


def test_large_tensor_sampled_blocks_match():
    import torch
    from synth.configs import DEPTHGRAFT_DECODE as cfg
    k = sgpu.make_device(cfg, "k")
    host = cfg.make("k", (9, 13, 2))
    got = k[9, 13, 2].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, host)
