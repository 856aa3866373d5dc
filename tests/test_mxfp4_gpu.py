"""MX FP4 expert weights (the mlx issue page's mode="mxfp4": 4-bit E2M1
codes, one E8M0 exponent byte per 32 values) through the C ABI, against the
oracle.

Bars: dequantised codes and fp32 weights bit-exact; the device generator's
bytes equal the host generator's.
"""
import numpy as np
import pytest

import oracle
from quantized_mixture_experts_affine_b200 import moeq, synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
SEED = 0


def test_mx_generator_and_dequant_bit_exact():
    d = synth.tensor_mx_dev(SEED, synth.tag(synth.UP, 40), 3, 72, 512)
    h = synth.tensor_mx_host(SEED, synth.tag(synth.UP, 40), 3, 72, 512)
    host = d.to_host()
    assert np.array_equal(host.w, h.w) and np.array_equal(host.s, h.s)
    t = moeq.qtensor(d.w, d.s, None, 72, 512, 4, 32, 3, moeq.FMT_MXFP4)
    for e in (0, 2):
        codes = torch.empty((72, 512), dtype=torch.uint8, device="cuda")
        w = torch.empty((72, 512), dtype=torch.float32, device="cuda")
        moeq.moeq_dequant(t, e, codes, w)
        torch.cuda.synchronize()
        assert np.array_equal(codes.cpu().numpy(), oracle.unpack(h, e))
        assert np.array_equal(w.cpu().numpy().view(np.uint32),
                              oracle.dequant_f32(h, e).view(np.uint32))
    assert moeq.moeq_device_status() == 0


def test_mx_every_code_and_scale_byte():
    """All 16 codes under exponent bytes 0 (2^-127, subnormal), 1, 100, 127,
    200 and 254 (6 * 2^127), bit-exact against the oracle."""
    codes = np.tile(np.arange(16, dtype=np.uint32), 2)
    w = np.zeros((6, 4), np.uint32)
    for j in range(8):
        w |= codes[j::8][None, :4] << (4 * j)
    ebytes = np.array([[0], [1], [100], [127], [200], [254]], np.uint8)
    host = synth.HostQ(w.reshape(1, 6, 4), ebytes.reshape(1, 6, 1), np.zeros(0, np.uint16),
                       6, 32, 4, 32, 1, 1)
    wd = torch.from_numpy(host.w.view(np.int32)).cuda()
    ed = torch.from_numpy(host.s).cuda()
    t = moeq.qtensor(wd, ed, None, 6, 32, 4, 32, 1, moeq.FMT_MXFP4)
    out = torch.empty((6, 32), dtype=torch.float32, device="cuda")
    moeq.moeq_dequant(t, 0, None, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint32),
                          oracle.dequant_f32(host).view(np.uint32))
