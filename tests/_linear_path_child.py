"""Child process for the oq_linear path test: OQ_LINEAR_PATH and OQ_GEMM_PAIR are read once per
process, so each GEMM form (in-GEMM decode of 4-bit activation codes; fp16 prepass into the
CTA-pair or the single-CTA GEMM) is exercised in a process of its own.  Checks oq_linear on uniform
random codes (every centroid used, ragged M and N tails) against the fp64 oracle, and the bf16
output against the fp32 output rounded to nearest even; exits non-zero on any failure."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle as O                                           # noqa: E402
from calibration_free_bit_b200 import oq                      # noqa: E402

LINEAR_RTOL = 1e-3


def main():
    worst = 0.0
    for ba, bw in [(4, 4), (4, 2), (4, 3), (4, 8)]:
        for T, N, d in [(200, 272, 384), (1, 16, 128), (129, 512, 1024), (300, 784, 3072),
                        (520, 528, 256)]:
            rng = np.random.default_rng(T * 7 + N + ba * 100 + bw + 5)
            xc = O.pack(rng.integers(0, 1 << ba, (T, d)).astype(np.uint8), ba)
            wc = O.pack(rng.integers(0, 1 << bw, (N, d)).astype(np.uint8), bw)
            s = rng.uniform(0.1, 50.0, T)
            rn = rng.uniform(0.5, 2.0, N)
            ca, cw = oq.oq_lloyd_max(d, ba), oq.oq_lloyd_max(d, bw)
            y = oq.oq_linear(ca, cw, torch.from_numpy(xc).cuda(),
                             torch.from_numpy(s.astype(np.float32)).cuda(),
                             torch.from_numpy(wc).cuda(),
                             torch.from_numpy(rn.astype(np.float32)).cuda())
            y16 = oq.oq_linear(ca, cw, torch.from_numpy(xc).cuda(),
                               torch.from_numpy(s.astype(np.float32)).cuda(),
                               torch.from_numpy(wc).cuda(),
                               torch.from_numpy(rn.astype(np.float32)).cuda(),
                               out_dtype=torch.bfloat16)
            oq.oq_check()
            if not torch.equal(y.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16)):
                print(f"FAIL bf16 output ba={ba} bw={bw} T={T} N={N} d={d}")
                return 1
            got = y.cpu().double().numpy()
            ref = O.linear(xc, s, wc, rn, d, ba, bw)
            err = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
            worst = max(worst, err)
            if not err <= LINEAR_RTOL:
                print(f"FAIL ba={ba} bw={bw} T={T} N={N} d={d}: rel_l2 {err}")
                return 1
    print(f"ok worst rel_l2 {worst:.3e}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
