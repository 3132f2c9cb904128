"""Child process for the fused-step test: OQ_FUSED_STEP is read once per process, so the
one-call path's persistent kernel (the quantize stage and the CTA-pair GEMM side by side) is
exercised in a process of its own.  Every case must equal oq_quantize_act + oq_linear bit for
bit (y and s); shapes outside the kernel's range, or with so few output tiles that the GEMM
splits its K loop, must take the other forms, still identical.
Exits non-zero on any failure."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from calibration_free_bit_b200 import oq, synth               # noqa: E402


def one(d, h, ba, bw, T, N, out, attn=False, seed=0):
    p = synth.get("flux_attn_w4a4")[0] if attn else synth.sweep_projection(d, 128, 4, T)
    x = synth.activations(p).cuda()
    W = (torch.randn(N, d, generator=torch.Generator().manual_seed(d + N + seed)) /
         d ** 0.5).cuda()
    r = oq.oq_build_rpbh(d, h, seed)
    ca, cw = oq.oq_lloyd_max(d, ba), oq.oq_lloyd_max(d, bw)
    wc, rn = oq.oq_quantize_weight(r, cw, W)
    xc, s_ref = oq.oq_quantize_act(r, ca, x)
    y_ref = oq.oq_linear(ca, cw, xc, s_ref, wc, rn, out_dtype=out)
    s = torch.empty(T, device="cuda")
    ys = [oq.oq_quantized_linear(r, ca, cw, x, wc, rn, s=s, out_dtype=out) for _ in range(2)]
    oq.oq_check()
    iv = torch.int32 if out == torch.float32 else torch.int16
    for y in ys:
        if not (torch.equal(s, s_ref) and torch.equal(y.view(iv), y_ref.view(iv))):
            diff = (y.float() - y_ref.float()).abs().max().item()
            print(f"FAIL d={d} h={h} A{ba} W{bw} T={T} N={N} {out}: max |dy| {diff}, "
                  f"s equal {torch.equal(s, s_ref)}")
            return False
    return True


def armed_wait():
    """The fused kernel's armed test wait: the call does its work, the wait runs out after its
    short limit and oq_check reports bit 0x10 of the fused kernel's error word; the outputs
    equal an unarmed call's and the next call is clean."""
    d, T, N = 1024, 2310, 784                  # enough tiles that the GEMM does not split K
    p = synth.sweep_projection(d, 128, 4, T)
    x = synth.activations(p).cuda()
    W = (torch.randn(N, d, generator=torch.Generator().manual_seed(3)) / d ** 0.5).cuda()
    r = oq.oq_build_rpbh(d, 128, 0)
    c4 = oq.oq_lloyd_max(d, 4)
    wc, rn = oq.oq_quantize_weight(r, c4, W)
    ref = oq.oq_quantized_linear(r, c4, c4, x, wc, rn)
    oq.oq_check()
    oq.oq_debug_arm_wait_timeout(oq.OQ_KERNEL_GEMM, 2_000_000)
    y = oq.oq_quantized_linear(r, c4, c4, x, wc, rn)
    try:
        oq.oq_check()
        print("FAIL armed wait not reported")
        return False
    except oq.OQError as e:
        if e.code != oq.OQ_EDEVICE or "fused=0x10 " not in str(e):
            print(f"FAIL armed wait reported as: {e}")
            return False
    y2 = oq.oq_quantized_linear(r, c4, c4, x, wc, rn)
    oq.oq_check()
    if not (torch.equal(y, ref) and torch.equal(y2, ref)):
        print("FAIL outputs around the armed wait differ")
        return False
    return True


def main():
    cases = [
        (3072, 128, 4, 4, 4608, 3072, torch.float32, True),    # the attention projection
        (3072, 128, 4, 4, 4608, 3072, torch.bfloat16, True),
        (1024, 64, 2, 4, 4099, 784, torch.float32, False),     # ragged T (odd) and N
        (2048, 256, 8, 2, 4353, 528, torch.float32, False),
        (4096, 128, 4, 8, 2310, 1040, torch.bfloat16, False),  # 8-bit weights: decode launch
        # few tiles (the GEMM splits its K loop) or outside the kernel: the other forms
        (3072, 128, 4, 4, 1, 16, torch.float32, False),        # one token
        (3072, 128, 4, 4, 2, 4096, torch.float32, False),
        (5120, 128, 4, 4, 64, 256, torch.float32, False),
    ]
    ok = True
    for d, h, ba, bw, T, N, out, attn in cases:
        ok = one(d, h, ba, bw, T, N, out, attn) and ok
    ok = armed_wait() and ok
    print("ok" if ok else "FAILED")
    return 0 if ok else 1


if __name__ == "__main__":
    sys.exit(main())
