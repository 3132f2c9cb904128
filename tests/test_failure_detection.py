"""Failure detection without a GPU fault.

Every wait inside liboq's kernels is bounded: a wait that runs out sets a bit in a device error
word, the kernel returns instead of hanging, and oq_check() reports OQ_EDEVICE with the bit.
oq_debug_arm_wait_timeout makes one such wait run out on purpose: the next launch of the chosen
kernel does its normal work and then waits on a shared-memory barrier that nothing completes,
with a short limit.  Nothing faults, traps or waits without a bound; the tests check that the
timeout is reported, that the outputs are those of an unarmed call, and that the context stays
usable for the calls that follow.  (The pages describe no failure handling; this covers the
library's own.)
"""
import ctypes as C

import numpy as np
import pytest
import torch

from calibration_free_bit_b200 import build as B
from calibration_free_bit_b200 import oq as oq_mod
from calibration_free_bit_b200 import synth

LIMIT = 2_000_000          # SM cycles: about 1 ms at the boost clock


def test_arming_validates_its_arguments():
    L = oq_mod.lib()
    assert L.oq_debug_arm_wait_timeout(2, LIMIT) == oq_mod.OQ_EINVAL     # the decode: no waits
    assert L.oq_debug_arm_wait_timeout(7, LIMIT) == oq_mod.OQ_EINVAL
    assert L.oq_debug_arm_wait_timeout(1, 999) == oq_mod.OQ_EINVAL
    assert L.oq_debug_arm_wait_timeout(3, 10 ** 10) == oq_mod.OQ_EINVAL
    assert b"limit_cycles" in L.oq_last_error()
    assert L.oq_debug_arm_wait_timeout(1, LIMIT) == oq_mod.OQ_OK
    assert L.oq_debug_arm_wait_timeout(0, 0) == oq_mod.OQ_OK             # disarm


@pytest.fixture(scope="module")
def oq(cuda_device):
    B.build()
    return oq_mod


def _inputs(oq, T=300, d=1024, N=272):
    p = synth.sweep_projection(d, 128, 4, T)
    x = synth.activations(p).cuda()
    W = (torch.randn(N, d, generator=torch.Generator().manual_seed(1)) / np.sqrt(d)).cuda()
    r = oq.oq_build_rpbh(d, 128, 0)
    ca, cw = oq.oq_lloyd_max(d, 4), oq.oq_lloyd_max(d, 4)
    return r, ca, cw, x, W


def _expect_device_error(oq, needle):
    with pytest.raises(oq.OQError) as e:
        oq.oq_check()
    assert e.value.code == oq.OQ_EDEVICE
    assert needle in str(e.value), str(e.value)


@pytest.mark.gpu
def test_quantize_wait_timeout_is_reported_and_recovered(oq):
    r, ca, _, x, _ = _inputs(oq)
    ref_codes, ref_s = oq.oq_quantize_act(r, ca, x)
    oq.oq_check()
    oq.oq_debug_arm_wait_timeout(oq.OQ_KERNEL_QUANTIZE, LIMIT)
    codes, s = oq.oq_quantize_act(r, ca, x)
    _expect_device_error(oq, "quantize=0x2 ")
    assert torch.equal(codes, ref_codes) and torch.equal(s, ref_s)
    # one-shot: the next call is clean, and the error word was cleared by oq_check
    codes2, s2 = oq.oq_quantize_act(r, ca, x)
    oq.oq_check()
    assert torch.equal(codes2, ref_codes) and torch.equal(s2, ref_s)


@pytest.mark.gpu
def test_gemm_wait_timeout_is_reported_and_recovered(oq):
    r, ca, cw, x, W = _inputs(oq)
    wc, rn = oq.oq_quantize_weight(r, cw, W)
    xc, s = oq.oq_quantize_act(r, ca, x)
    ref = oq.oq_linear(ca, cw, xc, s, wc, rn)
    oq.oq_check()
    oq.oq_debug_arm_wait_timeout(oq.OQ_KERNEL_GEMM, LIMIT)
    y = oq.oq_linear(ca, cw, xc, s, wc, rn)
    _expect_device_error(oq, "linear=0x8 ")
    assert torch.equal(y, ref)
    # the one-call path after the failure, then armed inside it as well
    y1 = oq.oq_quantized_linear(r, ca, cw, x, wc, rn)
    oq.oq_check()
    assert torch.equal(y1, ref)
    oq.oq_debug_arm_wait_timeout(oq.OQ_KERNEL_GEMM, LIMIT)
    y2 = oq.oq_quantized_linear(r, ca, cw, x, wc, rn)
    _expect_device_error(oq, "linear=0x8 ")
    assert torch.equal(y2, ref)


@pytest.mark.gpu
def test_disarm_before_launch(oq):
    r, ca, _, x, _ = _inputs(oq)
    oq.oq_debug_arm_wait_timeout(oq.OQ_KERNEL_QUANTIZE, LIMIT)
    oq.oq_debug_arm_wait_timeout(0, 0)
    oq.oq_quantize_act(r, ca, x)
    oq.oq_check()
