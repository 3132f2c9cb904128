"""oq_linear_noalloc: the codebook linear layer for callers that cannot allocate device memory.

Some callers can't call cudaMalloc: plug-ins hosted by a framework that owns all device memory
(and gives them no allocator), or serving loops that forbid allocation on the request path
because it can synchronise the device.  For them liboq keeps the linear layer's fp16 operand
workspace in a fixed array compiled into the library, and oq_linear_noalloc allocates nothing.

This file is collected last on purpose.  It checks, through the C ABI, that two calls in a
row give the same output as oq_linear (within the linear layer's parity tolerance), and that
a call needing more workspace than the fixed array is refused with a clear error.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from calibration_free_bit_b200 import build as B
from calibration_free_bit_b200 import synth

pytestmark = pytest.mark.gpu

LINEAR_RTOL = 1e-3


@pytest.fixture(scope="module")
def oq(cuda_device):
    B.build()
    from calibration_free_bit_b200 import oq as _oq
    return _oq


def _ptr(t):
    return C.c_void_p(t.data_ptr())


def test_noalloc_matches_oq_linear_on_two_calls(oq):
    p = synth.get("flux_attn_w4a4")[0]              # 4608 x 3072 -> 3072: 47 MB workspace
    r = oq.oq_build_rpbh(p.d, p.h, 0)
    ca, cw = oq.oq_lloyd_max(p.d, p.bits_a), oq.oq_lloyd_max(p.d, p.bits_w)
    xc, s = oq.oq_quantize_act(r, ca, synth.activations(p).cuda())
    wc, rn = oq.oq_quantize_weight(r, cw, synth.weight(p).cuda())
    ref = oq.oq_linear(ca, cw, xc, s, wc, rn)
    oq.oq_check()

    L = oq.lib()
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    outs = []
    for _ in range(2):
        y = torch.full((p.T, p.out), float("nan"), dtype=torch.float32, device="cuda")
        rc = L.oq_linear_noalloc(ca.handle, cw.handle, _ptr(xc), _ptr(s), _ptr(wc), _ptr(rn),
                                 p.T, p.d, p.out, _ptr(y), oq.OQ_F32, stream)
        assert rc == oq.OQ_OK, L.oq_last_error()
        oq.oq_check()
        outs.append(y)
    ref_np = ref.double().cpu().numpy()
    for y in outs:
        got = y.double().cpu().numpy()
        assert np.isfinite(got).all()
        err = np.linalg.norm(got - ref_np) / np.linalg.norm(ref_np)
        assert err <= LINEAR_RTOL, err


def test_noalloc_refuses_sizes_beyond_its_workspace(oq):
    d, T, N = 5120, 65520, 13824                     # ~800 MB of operands: over the limit
    ca = oq.oq_lloyd_max(d, 4)
    L = oq.lib()
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    rc = L.oq_linear_noalloc(ca.handle, ca.handle, _ptr(dummy), _ptr(dummy), _ptr(dummy),
                             _ptr(dummy), T, d, N, _ptr(dummy), oq.OQ_F32, None)
    assert rc == oq.OQ_EINVAL
    msg = L.oq_last_error().decode()
    assert "workspace" in msg and str(64 << 20) in msg
