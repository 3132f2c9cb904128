"""Child process for the oq_linear path test: OQ_LINEAR_PATH and OQ_GEMM_PAIR are read once per
process, so each GEMM form (in-GEMM decode of 4-bit activation or weight codes; fp16 prepass
into the CTA-pair or the single-CTA GEMM) is exercised in a process of its own.  Checks oq_linear on uniform
random codes (every centroid used, ragged M and N tails) against the fp64 oracle, and the bf16
output against the fp32 output rounded to nearest even, and oq_quantized_linear (which takes the
same form) against oq_quantize_act + oq_linear bit for bit; prints the SHA-256 of the attention
workload's y so that the forms can be compared with each other; exits non-zero on any
failure."""
import hashlib
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle as O                                           # noqa: E402
from calibration_free_bit_b200 import oq, synth               # noqa: E402

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
    # the one-call path in this process's form: bit-identical to the two calls, and its output
    # on the attention workload hashed so that the parent can compare the forms bit for bit
    p = synth.get("flux_attn_w4a4")[0]
    x = synth.activations(p).cuda()
    W = synth.weight(p).cuda()
    r = oq.oq_build_rpbh(p.d, p.h, 0)
    ca, cw = oq.oq_lloyd_max(p.d, 4), oq.oq_lloyd_max(p.d, 4)
    wc, rn = oq.oq_quantize_weight(r, cw, W)
    xc, s_ref = oq.oq_quantize_act(r, ca, x)
    y_ref = oq.oq_linear(ca, cw, xc, s_ref, wc, rn)
    for out in (torch.float32, torch.bfloat16):
        y_two = y_ref if out == torch.float32 else oq.oq_linear(ca, cw, xc, s_ref, wc, rn,
                                                                out_dtype=out)
        s1 = torch.empty(p.T, device="cuda")
        y1 = oq.oq_quantized_linear(r, ca, cw, x, wc, rn, s=s1, out_dtype=out)
        oq.oq_check()
        iv = torch.int32 if out == torch.float32 else torch.int16
        if not (torch.equal(s1, s_ref) and torch.equal(y1.view(iv), y_two.view(iv))):
            print(f"FAIL one-call path differs from the two calls ({out})")
            return 1
    for d, h, T, N in [(1024, 64, 129, 272), (2048, 128, 77, 40), (3072, 128, 9, 512)]:
        pp = synth.sweep_projection(d, h, 4, T)
        xx = synth.activations(pp).cuda()
        WW = (torch.randn(N, d, generator=torch.Generator().manual_seed(d)) / d ** 0.5).cuda()
        rr = oq.oq_build_rpbh(d, h, 0)
        c4 = oq.oq_lloyd_max(d, 4)
        wcc, rnn = oq.oq_quantize_weight(rr, c4, WW)
        xcc, ss = oq.oq_quantize_act(rr, c4, xx)
        y2 = oq.oq_linear(c4, c4, xcc, ss, wcc, rnn)
        y1 = oq.oq_quantized_linear(rr, c4, c4, xx, wcc, rnn)
        oq.oq_check()
        if not torch.equal(y1.view(torch.int32), y2.view(torch.int32)):
            print(f"FAIL one-call path d={d} h={h} T={T} N={N}")
            return 1
    digest = hashlib.sha256(y_ref.cpu().numpy().tobytes()).hexdigest()
    print(f"ok worst rel_l2 {worst:.3e}")
    print(f"yhash {digest}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
