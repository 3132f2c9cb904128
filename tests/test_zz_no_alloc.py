"""oq_linear_noalloc: the codebook linear layer for callers that cannot allocate device memory.

Some callers can't call cudaMalloc: plug-ins hosted by a framework that owns all device memory
(and gives them no allocator), or serving loops that forbid allocation on the request path
because it can synchronise the device.  For them liboq keeps the linear layer's fp16 operand
workspace in a fixed array compiled into the library, and oq_linear_noalloc allocates nothing.

The call runs exactly the kernels of oq_linear's default form (decode prepass, then the GEMM),
so its output must equal oq_linear's bit for bit; one case is also checked against the fp64
oracle on sampled outputs.  Calls go through the C ABI directly (ctypes), two in a row per
case, and a small ragged call follows a large one, so stale contents of the shared array
cannot leak into a later result.

The file name sorts last so that pytest collects it after every other test file: a run that
stops at the first failure (-x) has then already run the rest of the suite.  Nothing here
depends on the order; each case also passes in a fresh process on its own.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle as O
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


def _noalloc(oq, ca, cw, xc, s, wc, rn, T, d, N, out_dtype):
    L = oq.lib()
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    y = torch.full((T, N), float("nan"), dtype=out_dtype, device="cuda")
    rc = L.oq_linear_noalloc(ca.handle, cw.handle, _ptr(xc), _ptr(s), _ptr(wc), _ptr(rn),
                             T, d, N, _ptr(y),
                             oq.OQ_F32 if out_dtype == torch.float32 else oq.OQ_BF16, stream)
    assert rc == oq.OQ_OK, L.oq_last_error()
    oq.oq_check()
    return y


def _bits(y):
    return y.view(torch.int32 if y.dtype == torch.float32 else torch.int16)


def test_noalloc_matches_oq_linear_on_two_calls(oq):
    """The attention projection (4608 x 3072 -> 3072, 47 MB of workspace): two calls in a row
    are bit-identical to oq_linear, and sampled outputs are within the linear bound of the
    fp64 oracle on the same codes."""
    p = synth.get("flux_attn_w4a4")[0]
    r = oq.oq_build_rpbh(p.d, p.h, 0)
    ca, cw = oq.oq_lloyd_max(p.d, p.bits_a), oq.oq_lloyd_max(p.d, p.bits_w)
    xc, s = oq.oq_quantize_act(r, ca, synth.activations(p).cuda())
    wc, rn = oq.oq_quantize_weight(r, cw, synth.weight(p).cuda())
    ref = oq.oq_linear(ca, cw, xc, s, wc, rn)
    oq.oq_check()
    for _ in range(2):
        y = _noalloc(oq, ca, cw, xc, s, wc, rn, p.T, p.d, p.out, torch.float32)
        assert torch.equal(_bits(y), _bits(ref))
    rows = np.array([0, 1, 255, 256, 2047, 4095, 4607])
    cols = np.array([0, 7, 255, 256, 1500, 3071])
    got = y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()]
    want = O.linear(xc[rows.tolist()].cpu().numpy(), s[rows.tolist()].cpu().double().numpy(),
                    wc[cols.tolist()].cpu().numpy(), rn[cols.tolist()].cpu().double().numpy(),
                    p.d, p.bits_a, p.bits_w)
    err = np.linalg.norm(got.cpu().double().numpy() - want) / np.linalg.norm(want)
    assert err <= LINEAR_RTOL, err


@pytest.mark.parametrize("T,N,d,ba,bw,out_dtype", [
    (129, 272, 1024, 4, 4, torch.bfloat16),      # ragged T and N, bf16 y
    (1, 16, 384, 2, 8, torch.bfloat16),          # one token, the smallest N
    (200, 48, 3072, 8, 3, torch.float32),
])
def test_noalloc_small_ragged_after_large(oq, T, N, d, ba, bw, out_dtype):
    """A large call first fills the shared array; the small ragged calls that follow (random
    codes, every centroid used) must still equal oq_linear bit for bit, twice in a row."""
    big = synth.get("flux_attn_w4a4")[0]
    cb = oq.oq_lloyd_max(big.d, 4)
    g = torch.Generator().manual_seed(5)
    bxc = torch.randint(0, 256, (big.T, big.d // 2), generator=g, dtype=torch.uint8).cuda()
    bwc = torch.randint(0, 256, (big.out, big.d // 2), generator=g, dtype=torch.uint8).cuda()
    bs = torch.rand(big.T, generator=g).cuda() + 0.5
    brn = torch.rand(big.out, generator=g).cuda() + 0.5
    _noalloc(oq, cb, cb, bxc, bs, bwc, brn, big.T, big.d, big.out, torch.float32)

    rng = np.random.default_rng(T + N + d)
    xc = torch.from_numpy(O.pack(rng.integers(0, 1 << ba, (T, d)).astype(np.uint8), ba)).cuda()
    wc = torch.from_numpy(O.pack(rng.integers(0, 1 << bw, (N, d)).astype(np.uint8), bw)).cuda()
    s = torch.from_numpy(rng.uniform(0.1, 50.0, T).astype(np.float32)).cuda()
    rn = torch.from_numpy(rng.uniform(0.5, 2.0, N).astype(np.float32)).cuda()
    ca, cw = oq.oq_lloyd_max(d, ba), oq.oq_lloyd_max(d, bw)
    ref = oq.oq_linear(ca, cw, xc, s, wc, rn, out_dtype=out_dtype)
    oq.oq_check()
    for _ in range(2):
        y = _noalloc(oq, ca, cw, xc, s, wc, rn, T, d, N, out_dtype)
        assert torch.equal(_bits(y), _bits(ref))


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
