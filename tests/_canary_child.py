"""Child process for the guard-byte test: every public call writes its outputs into views of
larger device buffers whose leading and trailing 256 bytes hold a guard pattern.  Each call
runs twice, with the output regions first filled with 0x00 and then with 0xFF: the guards must
be intact after both, and the two results equal byte for byte (so every output byte was
written and none depends on what the buffer held before).  The forms selected by the
environment (OQ_LINEAR_PATH, OQ_GEMM_PAIR, OQ_FUSED_STEP, OQ_K1_PATH, read once per process)
are covered by running this script under each.  Exits non-zero on any failure."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from calibration_free_bit_b200 import oq, synth               # noqa: E402

GUARD = 256
PATTERN = 0xA5


class Guarded:
    """A device output of `shape` and `dtype` inside guard bytes."""

    def __init__(self, shape, dtype):
        self.shape, self.dtype = shape, dtype
        self.n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((GUARD + self.n + GUARD,), PATTERN, dtype=torch.uint8,
                              device="cuda")

    def view(self, fill):
        self.buf[GUARD:GUARD + self.n].fill_(fill)
        return self.buf[GUARD:GUARD + self.n].view(self.dtype).view(self.shape)

    def check(self, what):
        b = self.buf.cpu().numpy()
        if not ((b[:GUARD] == PATTERN).all() and (b[GUARD + self.n:] == PATTERN).all()):
            raise AssertionError(f"{what}: guard bytes overwritten")
        return b[GUARD:GUARD + self.n].copy()


def twice(what, outs, call):
    """Run call(*views) with 0x00- and 0xFF-filled outputs; compare and check guards."""
    results = []
    for fill in (0x00, 0xFF):
        views = [g.view(fill) for g in outs]
        call(*views)
        oq.oq_check()
        results.append([g.check(what) for g in outs])
    for a, b in zip(*results):
        if not np.array_equal(a, b):
            raise AssertionError(f"{what}: output bytes depend on the buffer's old contents")


def main():
    failures = []

    def run(what, fn):
        try:
            fn()
        except Exception as e:                     # report every case, then fail
            failures.append(f"{what}: {e}")

    # rotate + quantize: lockstep, named, padded and small-block groups, fp32 and bf16 rows,
    # packed widths 2..8, GELU
    for d, h, bits, T, f32, gelu in [(384, 128, 3, 37, False, False),
                                     (1024, 64, 4, 37, False, False),
                                     (3968, 128, 6, 19, False, False),
                                     (256, 4, 2, 9, False, False),
                                     (256, 64, 8, 33, True, False),
                                     (2048, 256, 4, 21, False, True)]:
        p = synth.sweep_projection(d, 128, 4, T)
        x = synth.activations(p).cuda()
        if f32:
            x = x.float()
        r, cb = oq.oq_build_rpbh(d, h, 0), oq.oq_lloyd_max(d, bits)
        outs = [Guarded((T, d * bits // 8), torch.uint8), Guarded((T,), torch.float32)]
        run(f"quantize_act d={d} h={h} b={bits}",
            lambda: twice(f"quantize_act d={d}", outs,
                          lambda c, s: oq.oq_quantize_act(r, cb, x, c, s, gelu=gelu)))
    # weights
    W = (torch.randn(20, 256, generator=torch.Generator().manual_seed(2)) / 16).cuda()
    r, cw = oq.oq_build_rpbh(256, 64, 0), oq.oq_lloyd_max(256, 4)
    outs = [Guarded((20, 128), torch.uint8), Guarded((20,), torch.float32)]
    run("quantize_weight", lambda: twice("quantize_weight", outs,
                                         lambda c, n: oq.oq_quantize_weight(r, cw, W, c, n)))
    # linear layer, the one-call path and the fixed-workspace call: ragged T and N, both y types
    for d, h, ba, bw, T, N, out in [(1024, 128, 4, 4, 77, 40, torch.float32),
                                    (1024, 128, 4, 4, 129, 272, torch.bfloat16),
                                    (3072, 128, 4, 2, 300, 264, torch.float32),
                                    (512, 128, 3, 4, 65, 20, torch.float32)]:
        p = synth.sweep_projection(d, 128, 4, T)
        x = synth.activations(p).cuda()
        Wd = (torch.randn(N, d, generator=torch.Generator().manual_seed(d + N)) /
              d ** 0.5).cuda()
        r = oq.oq_build_rpbh(d, h, 0)
        ca, cw = oq.oq_lloyd_max(d, ba), oq.oq_lloyd_max(d, bw)
        wc, rn = oq.oq_quantize_weight(r, cw, Wd)
        xc, s = oq.oq_quantize_act(r, ca, x)
        ys = Guarded((T, N), out)
        run(f"linear T={T} N={N}", lambda: twice(
            f"linear T={T} N={N}", [ys],
            lambda y: oq.oq_linear(ca, cw, xc, s, wc, rn, y=y, out_dtype=out)))
        run(f"linear_noalloc T={T} N={N}", lambda: twice(
            f"linear_noalloc T={T} N={N}", [ys],
            lambda y: oq.oq_linear_noalloc(ca, cw, xc, s, wc, rn, y)))
        ss = Guarded((T,), torch.float32)
        run(f"quantized_linear T={T} N={N}", lambda: twice(
            f"quantized_linear T={T} N={N}", [ys, ss],
            lambda y, s1: oq.oq_quantized_linear(r, ca, cw, x, wc, rn, y=y, s=s1,
                                                 out_dtype=out)))
    torch.cuda.synchronize()
    for f in failures:
        print("FAIL", f)
    print("ok" if not failures else "FAILED")
    return 1 if failures else 0


if __name__ == "__main__":
    sys.exit(main())
