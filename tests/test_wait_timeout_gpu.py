"""Device failure path without a fault: the bounded waits the library's
kernels use (an mbarrier phase that never completes, a flag that nothing
sets) run out after about two seconds each, report MOEQ_ERR_TIMEOUT through
the device status word, and the context stays usable: a decode call made
afterwards reports OK and matches the oracle.
"""
import numpy as np
import pytest

from helpers import check_layer_outputs
from quantized_mixture_experts_affine_b200 import moeq, synth
from quantized_mixture_experts_affine_b200.layer import CONFIGS, layer_forward, synthetic_layer

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
SEED = 0


def test_bounded_waits_time_out_and_context_survives():
    assert moeq.moeq_device_status() == moeq.OK  # read and clear
    moeq.moeq_selftest_wait_timeout()
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == moeq.ERR_TIMEOUT
    assert moeq.moeq_device_status() == moeq.OK  # the read cleared it

    cfg = CONFIGS["tiny"]
    L = synthetic_layer(cfg, SEED, 0)
    M = 3
    xb = synth.normal_bf16_host(SEED, synth.tag(synth.X, 0), M * cfg.H).reshape(M, cfg.H)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    y, idx, w = layer_forward(L, x, mode=moeq.MODE_DECODE)
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == moeq.OK
    check_layer_outputs(cfg, SEED, 0, xb, y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy())
