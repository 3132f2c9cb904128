"""Child process for the K1 path test: OQ_K1_PATH is read once per process, so the selected
rotate+quantize kernel (OQ_K1_PATH=tc: the tensor-core one) is exercised in a process of its
own on bf16 shapes it supports, flux-attention rows included.  Uses the parity rules of
test_gpu_parity; exits non-zero on any failure."""
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle as O                                           # noqa: E402
from calibration_free_bit_b200 import oq, synth               # noqa: E402
import test_gpu_parity as T                                   # noqa: E402


def main():
    for d, h, bits, n in [(3072, 128, 4, 101), (2048, 64, 8, 37), (1024, 256, 2, 29),
                          (2560, 32, 6, 17), (512, 128, 3, 9), (384, 128, 4, 1),
                          (3072, 256, 4, 64)]:
        p = synth.sweep_projection(d, 128, 4, n)
        x = synth.activations(p)
        r = oq.oq_build_rpbh(d, h, 0)
        cb = oq.oq_lloyd_max(d, bits)
        g, gs = T.k1_gpu(oq, r, cb, x)
        o, os_, _, ou = T.k1_oracle(x, h, bits)
        T.check_codes(g, o, ou, d, bits, f"{os.environ.get('OQ_K1_PATH')} d={d} h={h} b={bits}")
        np.testing.assert_allclose(gs, os_, rtol=T.NORM_RTOL)
    # the attention workload's rows, every one of them
    p = synth.get("flux_attn_w4a4")[0]
    x = synth.activations(p, rows=np.arange(0, p.T, 3))
    r = oq.oq_build_rpbh(p.d, p.h, 0)
    cb = oq.oq_lloyd_max(p.d, 4)
    g, gs = T.k1_gpu(oq, r, cb, x)
    o, os_, _, ou = T.k1_oracle(x, p.h, 4)
    T.check_codes(g, o, ou, p.d, 4, "flux attention rows")
    np.testing.assert_allclose(gs, os_, rtol=T.NORM_RTOL)
    print("ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
