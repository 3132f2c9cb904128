"""GPU parity: liboq's sm_100a kernels (through the C ABI) against the fp64 oracle.

Bars (rcap.io OrbitQuant summary, pseudocode block; tolerances from the benchmark spec of
the method):
  * packed layout bit-exact (GPU codes re-packed by the oracle reproduce the GPU bytes);
  * activation / weight codes: >= 99.99% identical, and every mismatch is a neighbour code
    with the fp64 unit value within 1e-5 sigma of the boundary between them (the kernel decides
    in fp32: butterfly, norm and fixed-point grid rounding together move a decision by at most
    about 5e-6 sigma, so only values that close to a boundary may land in the other cell);
  * norms s / row_norms: relative error <= 5e-6 (fp32 accumulation over d squares);
  * oq_linear on identical codes: relative L2 error <= 1e-3 against the fp64 triple loop.
Inputs are the seeded synthetic workloads of calibration_free_bit_b200.synth; large
workloads are checked on sampled rows / columns (the oracle computes those one by one) and
on properties that hold at any size (norm preservation, code range).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from calibration_free_bit_b200 import build as B
from calibration_free_bit_b200 import synth

pytestmark = pytest.mark.gpu

CODE_MATCH = 0.9999
BOUNDARY_TOL = 1e-5        # in sigma units (unit-codebook units)
NORM_RTOL = 5e-6
LINEAR_RTOL = 1e-3
BF16_REL = 2.0 ** -9       # round-to-nearest bf16: relative error bound per element


@pytest.fixture(scope="module")
def oq(cuda_device):
    B.build()
    from calibration_free_bit_b200 import oq as _oq
    return _oq


_HANDLES = {}
_ROWS = {}


def activations(p):
    """synth.activations(p) for all rows, keeping the last matrix: the large workloads take
    seconds to draw, and consecutive tests often read the same rows (projections that share
    their data seeds, e.g. one shape under two bit settings, share the matrix)."""
    key = (p.cfg, p.proj, p.T, p.d, p.dtype, p.outlier_count, p.outlier_scale, p.token_scale,
           p.gelu)
    if key not in _ROWS:
        _ROWS.clear()
        _ROWS[key] = synth.activations(p)
    return _ROWS[key]


def handles(oq, d, h, ba, bw, seed=0):
    key = (d, h, ba, bw, seed)
    if key not in _HANDLES:
        _HANDLES[key] = (oq.oq_build_rpbh(d, h, seed), oq.oq_lloyd_max(d, ba),
                         oq.oq_lloyd_max(d, bw))
    return _HANDLES[key]


def check_codes(gpu_packed, orc_packed, orc_u, d, bits, what, marginal="gauss",
                count_rule=True):
    """Code-parity rule on a block of rows; returns the number of mismatches.  count_rule:
    apply the 99.99 % bound (off only for inputs built to sit on a boundary)."""
    gpu_packed = np.ascontiguousarray(gpu_packed)
    gcodes = O.unpack(gpu_packed, d, bits)
    # layout: the oracle's packer reproduces the GPU's bytes exactly
    assert np.array_equal(O.pack(gcodes, bits), gpu_packed), f"{what}: packed layout"
    ocodes = O.unpack(orc_packed, d, bits)
    bad = np.argwhere(gcodes != ocodes)
    n = gcodes.size
    if count_rule:
        assert len(bad) <= (1 - CODE_MATCH) * n + 1e-9, f"{what}: {len(bad)} of {n} codes differ"
    _, t = O.codebook(bits, marginal, d)
    for r, k in bad:
        u = orc_u[r, k]
        j = int(np.argmin(np.abs(t - u)))
        assert abs(u - t[j]) <= BOUNDARY_TOL, f"{what}: row {r} col {k} u={u} not near a boundary"
        assert {int(gcodes[r, k]), int(ocodes[r, k])} == {j, j + 1}, f"{what}: non-adjacent"
    return len(bad)


def k1_gpu(oq, r, cb, x_cpu, weight=False):
    x = x_cpu.cuda()
    fn = oq.oq_quantize_weight if weight else oq.oq_quantize_act
    codes, s = fn(r, cb, x)
    oq.oq_check()
    return codes.cpu().numpy(), s.cpu().numpy().astype(np.float64)


def k1_oracle(x_cpu, h, bits, weight=False, seed=0, marginal="gauss", permute=True):
    d = x_cpu.shape[1]
    perm, sign = (O.build_rpbh if permute else O.build_block_rht)(d, seed)
    x64 = x_cpu.double().numpy()
    fn = O.quantize_weight if weight else O.quantize_act
    return fn(x64, h, perm, sign, bits, detail=True, marginal=marginal)


# ----------------------------------------------------------------------------------------
# K1: rotate + norm + quantize
# ----------------------------------------------------------------------------------------

def test_k1_toy_fp32_activations_and_weights(oq):
    p = synth.get("toy_w4a4")[0]
    r, ca, cw = handles(oq, p.d, p.h, p.bits_a, p.bits_w)
    x, W = synth.activations(p), synth.weight(p)
    g, gs = k1_gpu(oq, r, ca, x)
    o, os_, _, ou = k1_oracle(x, p.h, p.bits_a)
    check_codes(g, o, ou, p.d, p.bits_a, "toy x")
    np.testing.assert_allclose(gs, os_, rtol=NORM_RTOL)
    g, gs = k1_gpu(oq, r, cw, W, weight=True)
    o, os_, _, ou = k1_oracle(W, p.h, p.bits_w, weight=True)
    check_codes(g, o, ou, p.d, p.bits_w, "toy W")
    np.testing.assert_allclose(gs, os_, rtol=NORM_RTOL)


@pytest.mark.parametrize("h", [32, 64, 128, 256, 512, 1024])
@pytest.mark.parametrize("bits", [2, 3, 4, 6, 8])
def test_k1_every_block_size_and_bit_width(oq, h, bits):
    d = 2048 if h <= 512 else 3072
    T = 37                                  # odd: the last token pair has one token
    p = synth.sweep_projection(d, 128, 4, T)
    x = synth.activations(p)
    r = oq.oq_build_rpbh(d, h, 0)
    cb = oq.oq_lloyd_max(d, bits)
    g, gs = k1_gpu(oq, r, cb, x)
    o, os_, _, ou = k1_oracle(x, h, bits)
    check_codes(g, o, ou, d, bits, f"h={h} b={bits}")
    np.testing.assert_allclose(gs, os_, rtol=NORM_RTOL)


@pytest.mark.parametrize("d,h,bits,T", [
    (896, 128, 4, 301),      # 28 position threads a pair: one warp, 4 padding lanes
    (3968, 128, 2, 257),     # 124 threads: four warps, the last with 28
    (3968, 64, 8, 64),       # fewer pairs than SMs
    (9728, 256, 6, 101),     # the text encoder's down input: 304 threads in 10 warps
    (13824, 128, 4, 67),     # the video FFN's down input: 432 threads in 14 warps
])
def test_k1_groups_padded_to_whole_warps(oq, d, h, bits, T):
    """bf16 widths whose d/32 position threads a token pair are not a whole number of warps
    but waste at most one lane in eight run the named-barrier K1 with each group padded to
    whole warps (the padding lanes own no positions): codes and norms against the oracle,
    bf16 input with outlier channels, odd T."""
    p = synth.sweep_projection(d, 128, 4, T)
    x = synth.activations(p)
    r = oq.oq_build_rpbh(d, h, 0)
    cb = oq.oq_lloyd_max(d, bits)
    g, gs = k1_gpu(oq, r, cb, x)
    o, os_, _, ou = k1_oracle(x, h, bits)
    check_codes(g, o, ou, d, bits, f"d={d} h={h} b={bits}")
    np.testing.assert_allclose(gs, os_, rtol=NORM_RTOL)


@pytest.mark.parametrize("d,h,bits", [(128, 64, 2), (128, 128, 4), (256, 64, 8), (384, 128, 3)])
def test_exact_marginal_codebook_k1_and_linear(oq, d, h, bits):
    """The f_d codebook (oq_lloyd_max_marginal, OQ_MARGINAL_EXACT) through K1 and the linear
    layer, at the small d where it differs most from N(0, 1/d)."""
    T, N = 150, 272
    p = synth.sweep_projection(d, h, 4, T)
    x = synth.activations(p)
    W = torch.randn(N, d, generator=torch.Generator().manual_seed(d + bits)) / math.sqrt(d)
    r = oq.oq_build_rpbh(d, h, 0)
    cb = oq.oq_lloyd_max(d, bits, "exact")
    g, gs = k1_gpu(oq, r, cb, x)
    o, os_, _, ou = k1_oracle(x, h, bits, marginal="sphere")
    check_codes(g, o, ou, d, bits, f"exact d={d} b={bits}", marginal="sphere")
    np.testing.assert_allclose(gs, os_, rtol=NORM_RTOL)
    gw, gws = k1_gpu(oq, r, cb, W, weight=True)
    ow, ows, _, wu = k1_oracle(W, h, bits, weight=True, marginal="sphere")
    check_codes(gw, ow, wu, d, bits, f"exact W d={d} b={bits}", marginal="sphere")
    y = linear_gpu(oq, cb, cb, o, os_, ow, ows)
    ref = O.linear(o, os_, ow, ows, d, bits, bits, marginal="sphere")
    assert rel_l2(y, ref) <= LINEAR_RTOL


def test_block_rht_k1_and_linear(oq):
    """The Block-RHT ablation (identity permutation) through K1 and the linear layer on sampled
    rows of the attention workload, and on an input concentrated on one block of positions,
    which Block-RHT leaves concentrated."""
    p = synth.get("flux_attn_w4a4")[0]
    rows = np.arange(0, p.T, 53)
    x = synth.activations(p, rows=rows)
    rng = np.random.default_rng(1)
    adv = np.zeros((9, p.d), np.float32)
    adv[:, p.h:2 * p.h] = rng.standard_normal((9, p.h))
    x = torch.cat([x, torch.from_numpy(adv).to(x.dtype)])
    r = oq.oq_build_block_rht(p.d, p.h, 0)
    ca, cw = oq.oq_lloyd_max(p.d, 4), oq.oq_lloyd_max(p.d, 4)
    g, gs = k1_gpu(oq, r, ca, x)
    o, os_, _, ou = k1_oracle(x, p.h, 4, permute=False)
    check_codes(g, o, ou, p.d, 4, "block-rht x")
    np.testing.assert_allclose(gs, os_, rtol=NORM_RTOL)
    half = 1 << 3                                     # code of 0: the block stays local
    codes = O.unpack(g[-9:], p.d, 4)
    assert np.all(codes[:, :p.h] == half) and np.all(codes[:, 2 * p.h:] == half)
    W = synth.weight(p)[:272]
    gw, gws = k1_gpu(oq, r, cw, W, weight=True)
    y = linear_gpu(oq, ca, cw, g, gs, gw, gws)
    ref = O.linear(g, gs, gw, gws, p.d, 4, 4)
    assert rel_l2(y, ref) <= LINEAR_RTOL


def test_k1_flux_attention_full_size(oq):
    """4608 x 3072 bf16, W4A4, h=128: every row against the oracle."""
    p = synth.get("flux_attn_w4a4")[0]
    r, ca, cw = handles(oq, p.d, p.h, p.bits_a, p.bits_w)
    x = synth.activations(p)
    g, gs = k1_gpu(oq, r, ca, x)
    o, os_, _, ou = k1_oracle(x, p.h, p.bits_a)
    check_codes(g, o, ou, p.d, p.bits_a, "flux attn x")
    np.testing.assert_allclose(gs, os_, rtol=NORM_RTOL)
    W = synth.weight(p)
    g, gs = k1_gpu(oq, r, cw, W, weight=True)
    o, os_, _, ou = k1_oracle(W, p.h, p.bits_w, weight=True)
    check_codes(g, o, ou, p.d, p.bits_w, "flux attn W")
    np.testing.assert_allclose(gs, os_, rtol=NORM_RTOL)


def test_k1_edge_rows(oq):
    """Zero rows, a single huge outlier, a one-hot row, tiny values, T = 1 and T = 0.
    (Rows below ~1e-17 would underflow fp32 squares; 1e-15 is still exact in fp32.)"""
    d, h, bits = 1024, 128, 4
    r = oq.oq_build_rpbh(d, h, 0)
    cb = oq.oq_lloyd_max(d, bits)
    x = torch.zeros((7, d), dtype=torch.bfloat16)
    x[1, 5] = 1.0
    x[2] = torch.randn(d, generator=torch.Generator().manual_seed(3)).bfloat16()
    x[2, 17] = 3.0e4
    x[3] = 1e-15
    x[5, :] = -2.0
    g, gs = k1_gpu(oq, r, cb, x)
    o, os_, _, ou = k1_oracle(x, h, bits)
    check_codes(g, o, ou, d, bits, "edge rows")
    np.testing.assert_allclose(gs, os_, rtol=NORM_RTOL, atol=0)
    assert gs[0] == 0.0 and gs[4] == 0.0 and gs[6] == 0.0
    assert np.all(O.unpack(g[[0, 4, 6]], d, bits) == 8)
    # T = 1
    g1, s1 = k1_gpu(oq, r, cb, x[2:3])
    assert np.array_equal(g1[0], g[2]) and s1[0] == gs[2]
    # T = 0 is a no-op
    codes, s = oq.oq_quantize_act(r, cb, torch.empty((0, d), dtype=torch.bfloat16,
                                                      device="cuda"))
    assert codes.shape == (0, d // 2) and s.shape == (0,)


def test_k1_max_dimension(oq):
    """d = 16384 (the sweep's largest), h = 256 and 128, bf16 and fp32 inputs."""
    p = synth.sweep_projection(16384, 256, 8, 64)
    x = synth.activations(p)
    for h, bits, xin in [(256, 8, x), (128, 4, x.float()), (256, 3, x.float())]:
        r = oq.oq_build_rpbh(16384, h, 0)
        cb = oq.oq_lloyd_max(16384, bits)
        g, gs = k1_gpu(oq, r, cb, xin)
        o, os_, _, ou = k1_oracle(xin, h, bits)
        check_codes(g, o, ou, 16384, bits, f"d=16384 h={h} b={bits}")
        np.testing.assert_allclose(gs, os_, rtol=NORM_RTOL)


def test_k1_video_ffn_full_size_sampled(oq):
    """65520 x 13824 bf16 (down projection input, W4A8): all rows on the GPU in the launch
    configuration the benchmark uses; sampled rows against the oracle, every norm against
    ||x|| (the rotation preserves norms)."""
    p = synth.get("video_ffn_w4a8")[1]
    r, ca, _ = handles(oq, p.d, p.h, p.bits_a, p.bits_w)
    x = activations(p)
    xg = x.cuda()
    codes, s = oq.oq_quantize_act(r, ca, xg)
    oq.oq_check()
    norm_ref = np.concatenate([torch.linalg.vector_norm(x[i:i + 4096].double(), dim=1).numpy()
                               for i in range(0, p.T, 4096)])
    np.testing.assert_allclose(s.cpu().double().numpy(), norm_ref, rtol=NORM_RTOL)
    rows = np.array([0, 1, 17, 32759, 32760, 40000, 65519])
    o, os_, _, ou = k1_oracle(x[rows], p.h, p.bits_a)
    check_codes(codes[rows].cpu().numpy(), o, ou, p.d, p.bits_a, "video ffn sampled")


# ----------------------------------------------------------------------------------------
# K2: codebook linear layer
# ----------------------------------------------------------------------------------------

def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def linear_gpu(oq, ca, cw, xc, s, wc, rn):
    dev = "cuda"
    y = oq.oq_linear(ca, cw, torch.from_numpy(np.ascontiguousarray(xc)).to(dev),
                     torch.from_numpy(np.asarray(s, np.float32)).to(dev),
                     torch.from_numpy(np.ascontiguousarray(wc)).to(dev),
                     torch.from_numpy(np.asarray(rn, np.float32)).to(dev))
    oq.oq_check()
    return y.cpu().double().numpy()


def test_linear_toy_on_oracle_codes(oq):
    p = synth.get("toy_w4a4")[0]
    _, ca, cw = handles(oq, p.d, p.h, p.bits_a, p.bits_w)
    xc, s, _, _ = k1_oracle(synth.activations(p), p.h, p.bits_a)
    wc, rn, _, _ = k1_oracle(synth.weight(p), p.h, p.bits_w, weight=True)
    y = linear_gpu(oq, ca, cw, xc, s, wc, rn)
    ref = O.linear(xc, s, wc, rn, p.d, p.bits_a, p.bits_w)
    assert rel_l2(y, ref) <= LINEAR_RTOL


@pytest.mark.parametrize("ba,bw", [(4, 4), (4, 2), (4, 3), (3, 4), (2, 2), (8, 4), (2, 8), (8, 8),
                                   (3, 2), (6, 6), (4, 6)])
@pytest.mark.parametrize("T,N,d", [(200, 272, 384), (1, 16, 128), (129, 512, 1024)])
def test_linear_random_codes_ragged(oq, ba, bw, T, N, d):
    """Uniform random codes (every centroid used), ragged M and N tails."""
    rng = np.random.default_rng(T * 7 + N + ba * 100 + bw)
    xc = O.pack(rng.integers(0, 1 << ba, (T, d)).astype(np.uint8), ba)
    wc = O.pack(rng.integers(0, 1 << bw, (N, d)).astype(np.uint8), bw)
    s = rng.uniform(0.1, 50.0, T)
    rn = rng.uniform(0.5, 2.0, N)
    ca, cw = oq.oq_lloyd_max(d, ba), oq.oq_lloyd_max(d, bw)
    y = linear_gpu(oq, ca, cw, xc, s, wc, rn)
    ref = O.linear(xc, s, wc, rn, d, ba, bw)
    assert rel_l2(y, ref) <= LINEAR_RTOL


def _sampled_linear(oq, p, rows, cols):
    """Full-size GPU path (K1 on all of x and W, then oq_linear), with the sampled rows of
    x_codes/s and of W_codes/row_norms replaced by the oracle's, so that the compared
    outputs y[rows, cols] come from identical codes."""
    r, ca, cw = handles(oq, p.d, p.h, p.bits_a, p.bits_w)
    x = activations(p)
    W = synth.weight(p)
    xc, s = oq.oq_quantize_act(r, ca, x.cuda())
    wc, rn = oq.oq_quantize_weight(r, cw, W.cuda())
    oq.oq_check()
    oxc, os_, _, ou = k1_oracle(x[rows], p.h, p.bits_a)
    owc, orn, _, wu = k1_oracle(W[cols], p.h, p.bits_w, weight=True)
    check_codes(xc[rows].cpu().numpy(), oxc, ou, p.d, p.bits_a, p.name + " x")
    check_codes(wc[cols].cpu().numpy(), owc, wu, p.d, p.bits_w, p.name + " W")
    ri, ci = torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()
    xc[ri] = torch.from_numpy(oxc).cuda()
    s[ri] = torch.from_numpy(os_.astype(np.float32)).cuda()
    wc[ci] = torch.from_numpy(owc).cuda()
    rn[ci] = torch.from_numpy(orn.astype(np.float32)).cuda()
    y = oq.oq_linear(ca, cw, xc, s, wc, rn)
    oq.oq_check()
    got = y[ri][:, ci].cpu().double().numpy()
    ref = O.linear(oxc, os_, owc, orn, p.d, p.bits_a, p.bits_w)
    assert rel_l2(got, ref) <= LINEAR_RTOL, rel_l2(got, ref)
    return y


def test_linear_flux_attention_full_size(oq):
    p = synth.get("flux_attn_w4a4")[0]
    rows = np.unique(np.concatenate([np.arange(0, 4608, 97), [4607, 4095, 4096]]))
    cols = np.unique(np.concatenate([np.arange(0, 3072, 41), [3071]]))
    _sampled_linear(oq, p, rows, cols)


@pytest.mark.parametrize("which", [0, 1])
def test_linear_flux_mlp_full_size(oq, which):
    p = synth.get("flux_mlp_w2a4")[which]
    rows = np.arange(0, p.T, 151)
    cols = np.arange(3, p.out, 389)
    _sampled_linear(oq, p, rows, cols)


@pytest.mark.parametrize("variant", ["video_ffn_w3a4", "video_ffn_w4a8"])
def test_linear_video_ffn_up_full_size(oq, variant):
    p = synth.get(variant)[0]
    rows = np.array([0, 5, 32759, 32760, 50000, 65408, 65519])
    cols = np.arange(11, p.out, 977)
    _sampled_linear(oq, p, rows, cols)


def test_linear_path_selection(oq):
    """Every GEMM form against the oracle, each in a child process (the variables are read
    once per process): the fp16 prepass feeding the CTA-pair GEMM (default), the same prepass
    feeding the single-CTA GEMM (OQ_GEMM_PAIR=0), 4-bit activation codes decoded inside the
    CTA-pair GEMM (OQ_LINEAR_PATH=fused) or the single-CTA one (both variables), and 4-bit
    weight codes decoded inside the CTA-pair GEMM (OQ_LINEAR_PATH=wcodes; with
    OQ_GEMM_PAIR=0 that form does not apply and the prepass serves the weights).  In each,
    oq_quantized_linear takes the same form and equals the two calls bit for bit, and the
    attention workload's y is identical across all forms (same fp16 operands, same MMA
    order)."""
    import os
    import re
    import subprocess
    import sys
    child = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_linear_path_child.py")
    hashes = {}
    for path in ("default", "fused", "single", "fused_single", "wcodes", "wcodes_single"):
        env = dict(os.environ)
        env.pop("OQ_LINEAR_PATH", None)
        env.pop("OQ_GEMM_PAIR", None)
        if path.startswith("fused"):
            env["OQ_LINEAR_PATH"] = "fused"
        if path.startswith("wcodes"):
            env["OQ_LINEAR_PATH"] = "wcodes"
        if path.endswith("single"):
            env["OQ_GEMM_PAIR"] = "0"
        r = subprocess.run([sys.executable, child], env=env, capture_output=True, text=True,
                           timeout=600)
        assert r.returncode == 0, path + ": " + r.stdout + r.stderr
        hashes[path] = re.search(r"yhash ([0-9a-f]+)", r.stdout).group(1)
    assert len(set(hashes.values())) == 1, hashes


def test_outputs_stay_inside_their_buffers(oq):
    """Guard bytes around every output buffer (the stand-in for a bounds sanitizer): each
    public call, on ragged shapes, writes only inside its outputs and writes all of them,
    under every form the environment selects (child processes; the variables are read once
    per process)."""
    import os
    import subprocess
    import sys
    child = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_canary_child.py")
    forms = {"default": {}, "acodes": {"OQ_LINEAR_PATH": "fused"},
             "wcodes": {"OQ_LINEAR_PATH": "wcodes"}, "single": {"OQ_GEMM_PAIR": "0"},
             "fused_step": {"OQ_FUSED_STEP": "1"}, "k1_tc": {"OQ_K1_PATH": "tc"}}
    for name, extra in forms.items():
        env = dict(os.environ)
        for k in ("OQ_LINEAR_PATH", "OQ_GEMM_PAIR", "OQ_FUSED_STEP", "OQ_K1_PATH",
                  "OQ_FUSED_RAMP"):
            env.pop(k, None)
        env.update(extra)
        r = subprocess.run([sys.executable, child], env=env, capture_output=True, text=True,
                           timeout=600)
        assert r.returncode == 0, name + ": " + r.stdout + r.stderr


def test_fused_step_matches_the_two_calls(oq):
    """OQ_FUSED_STEP=1: oq_quantized_linear as one persistent kernel (the rotate+quantize stage
    and the CTA-pair GEMM side by side, rows handed over per 256-row block) equals
    oq_quantize_act + oq_linear bit for bit on every supported shape tried, ragged T and N, one
    token, bf16 y and two calls in a row; a shape outside its range takes the other forms.
    Without ramp groups (the default) and with them (OQ_FUSED_RAMP=2: the GEMM warps first
    quantize two token pairs a group in the stage ring).  Runs in child processes (the
    variables are read once per process)."""
    import os
    import subprocess
    import sys
    child = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_fused_step_child.py")
    for ramp in ("0", "2"):                  # without and with ramp groups
        env = dict(os.environ, OQ_FUSED_STEP="1", OQ_FUSED_RAMP=ramp)
        env.pop("OQ_LINEAR_PATH", None)
        r = subprocess.run([sys.executable, child], env=env, capture_output=True, text=True,
                           timeout=600)
        assert r.returncode == 0, f"OQ_FUSED_RAMP={ramp}: " + r.stdout + r.stderr


@pytest.mark.parametrize("ba,bw", [(4, 4), (2, 8)])
@pytest.mark.parametrize("T,N,d", [(200, 272, 384), (129, 784, 1024)])
def test_linear_bf16_output(oq, ba, bw, T, N, d):
    """out_dtype bf16: every element is the fp32 result rounded to nearest even (the same
    epilogue arithmetic), so bf16(y_f32) == y_bf16 bit for bit, and the oracle bound widens by
    at most the rounding bound 2^-9."""
    rng = np.random.default_rng(T + 3 * N + ba)
    xc = O.pack(rng.integers(0, 1 << ba, (T, d)).astype(np.uint8), ba)
    wc = O.pack(rng.integers(0, 1 << bw, (N, d)).astype(np.uint8), bw)
    s = rng.uniform(0.1, 50.0, T)
    rn = rng.uniform(0.5, 2.0, N)
    ca, cw = oq.oq_lloyd_max(d, ba), oq.oq_lloyd_max(d, bw)
    args = [torch.from_numpy(xc).cuda(), torch.from_numpy(s.astype(np.float32)).cuda(),
            torch.from_numpy(wc).cuda(), torch.from_numpy(rn.astype(np.float32)).cuda()]
    y32 = oq.oq_linear(ca, cw, *args)
    y16 = oq.oq_linear(ca, cw, *args, out_dtype=torch.bfloat16)
    oq.oq_check()
    assert y16.dtype == torch.bfloat16
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))
    ref = O.linear(xc, s, wc, rn, d, ba, bw)
    assert rel_l2(y16.cpu().double().numpy(), ref) <= LINEAR_RTOL + BF16_REL


def test_linear_bf16_output_full_size(oq):
    """The attention projection at full size with bf16 y: bit-identical to rounding the fp32
    output of the same call."""
    p = synth.get("flux_attn_w4a4")[0]
    r, ca, cw = handles(oq, p.d, p.h, p.bits_a, p.bits_w)
    xc, s = oq.oq_quantize_act(r, ca, synth.activations(p).cuda())
    wc, rn = oq.oq_quantize_weight(r, cw, synth.weight(p).cuda())
    y32 = oq.oq_linear(ca, cw, xc, s, wc, rn)
    y16 = oq.oq_linear(ca, cw, xc, s, wc, rn, out_dtype=torch.bfloat16)
    oq.oq_check()
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))


@pytest.mark.parametrize("bits,h,d,T", [(4, 128, 12288, 40), (2, 128, 3072, 37),
                                        (8, 64, 1024, 33), (6, 256, 2048, 31),
                                        (3, 32, 512, 29)])
def test_k1_fused_gelu(oq, bits, h, d, T):
    """oq_quantize_act_gelu: codes and norms of R GELU(x) against the oracle's fp64 GELU, on
    pre-activations with outlier channels and a per-token lognormal scale (so GELU sees both
    large positive and large negative arguments)."""
    p = synth.sweep_projection(d, 128, 4, T)
    g = torch.Generator().manual_seed(d + bits)
    u = (synth.activations(p).float() * torch.exp(torch.randn(T, 1, generator=g))).to(
        torch.bfloat16)
    r = oq.oq_build_rpbh(d, h, 0)
    cb = oq.oq_lloyd_max(d, bits)
    xc, s = oq.oq_quantize_act(r, cb, u.cuda(), gelu=True)
    oq.oq_check()
    perm, sign = O.build_rpbh(d, 0)
    o, os_, _, ou = O.quantize_act(u.double().numpy(), h, perm, sign, bits, detail=True,
                                   gelu_input=True)
    check_codes(xc.cpu().numpy(), o, ou, d, bits, f"gelu d={d} b={bits}")
    np.testing.assert_allclose(s.cpu().numpy(), os_, rtol=NORM_RTOL)


@pytest.mark.parametrize("h", [64, 256])
def test_k1_fused_gelu_edge_values(oq, h):
    """The fused GELU at the values where its evaluation changes form: zero, values below and
    at the low end of its table (2^-16), inside it, at its top end (the largest bf16 below 16)
    and beyond (16 and up, both signs), mixed with N(0, 1) values so that the rows have
    ordinary norms.  Codes under the boundary-distance rule (such rows put many rotated values
    near a few points, as the small-block GELU case does) and norms against the oracle."""
    T, d, bits = 64, 1024, 4
    special = np.array([0.0, 1e-6, 2.0 ** -17, 2.0 ** -16, 1.5 * 2.0 ** -16, 0.004, 0.75,
                        1.0, 3.5, 15.9375, 16.0, 17.0, 100.0, 1e4])
    special = np.concatenate([special, -special])
    rng = np.random.default_rng(h)
    x = rng.standard_normal((T, d))
    mask = rng.random((T, d)) < 0.5
    x[mask] = rng.choice(special, size=int(mask.sum()))
    u = torch.from_numpy(x).float().to(torch.bfloat16)
    r = oq.oq_build_rpbh(d, h, 0)
    cb = oq.oq_lloyd_max(d, bits)
    xc, s = oq.oq_quantize_act(r, cb, u.cuda(), gelu=True)
    oq.oq_check()
    perm, sign = O.build_rpbh(d, 0)
    o, os_, _, ou = O.quantize_act(u.double().numpy(), h, perm, sign, bits, detail=True,
                                   gelu_input=True)
    check_codes(xc.cpu().numpy(), o, ou, d, bits, f"gelu edges h={h}", count_rule=False)
    np.testing.assert_allclose(s.cpu().numpy(), os_, rtol=NORM_RTOL)


def test_k1_fused_gelu_rejects_fp32(oq):
    r, cb = oq.oq_build_rpbh(256, 64, 0), oq.oq_lloyd_max(256, 4)
    with pytest.raises(oq.OQError):
        oq.oq_quantize_act(r, cb, torch.zeros(4, 256, device="cuda"), gelu=True)


def test_k1_tensor_core_path(oq):
    """With OQ_K1_PATH=tc, bf16 rows with h <= 256 and d up to ~3.9K go to the tensor-core
    K1 (block transform as tcgen05.mma); a child process (the variable is read once per
    process) checks it against the oracle under the same rules, on every supported h and
    bit width, ragged tiles included."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, OQ_K1_PATH="tc")
    child = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_k1_path_child.py")
    r = subprocess.run([sys.executable, child], env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout + r.stderr



@pytest.mark.parametrize("d,h,ba,bw,T,N,gelu,out", [
    (3072, 128, 4, 4, 4608, 3072, False, torch.float32),    # the attention projection
    (384, 128, 4, 2, 37, 272, False, torch.float32),        # ragged T and N
    (1024, 64, 2, 8, 129, 512, False, torch.bfloat16),
    (2048, 256, 8, 4, 33, 160, False, torch.float32),
    (1024, 128, 3, 4, 65, 256, False, torch.float32),       # fallback: codes + decode
    (2560, 128, 6, 6, 50, 336, False, torch.float32),       # fallback: 6-bit
    (2048, 512, 4, 4, 40, 128, False, torch.float32),       # fallback: h = 512
    (3072, 128, 4, 2, 100, 384, True, torch.float32),       # GELU pre-activation
    (1024, 64, 2, 4, 64, 48, False, torch.bfloat16),        # fused decode, 32 pairs < SMs
    (2048, 128, 2, 2, 400, 400, False, torch.float32),      # fused 2-bit weight decode
    (3072, 128, 4, 4, 17, 16, True, torch.float32),         # fused decode, odd T, GELU
    (3072, 128, 4, 4, 1, 16, False, torch.float32),         # N > T: decode beside K1
    (3968, 128, 4, 4, 300, 256, False, torch.float32),      # fused decode, padded groups
    (896, 64, 8, 2, 77, 48, False, torch.bfloat16),         # the same, one warp a group
])
def test_quantized_linear_matches_the_two_calls(oq, d, h, ba, bw, T, N, gelu, out):
    """oq_quantized_linear (x -> y, codes never in memory) is bit-identical to
    oq_quantize_act (or _gelu) followed by oq_linear: y and the norms s.  With 2- or 4-bit
    weights, 2/4/8-bit activations, the named-barrier K1 (d/32 threads a pair in whole warps,
    or padded to them), d <= 5120 and N <= T the weight
    decode runs inside K1 (also when there are fewer token pairs than SMs, and with groups
    padded to whole warps); the other rows take the side-stream decode."""
    p = synth.sweep_projection(d, 128, 4, T) if d != 3072 or T != 4608 else \
        synth.get("flux_attn_w4a4")[0]
    x = synth.activations(p).cuda()
    W = (torch.randn(N, d, generator=torch.Generator().manual_seed(d + N)) /
         math.sqrt(d)).cuda()
    r = oq.oq_build_rpbh(d, h, 0)
    ca, cw = oq.oq_lloyd_max(d, ba), oq.oq_lloyd_max(d, bw)
    wc, rn = oq.oq_quantize_weight(r, cw, W)
    xc, s_ref = oq.oq_quantize_act(r, ca, x, gelu=gelu)
    y_ref = oq.oq_linear(ca, cw, xc, s_ref, wc, rn, out_dtype=out)
    s = torch.empty(T, device="cuda")
    y = oq.oq_quantized_linear(r, ca, cw, x, wc, rn, s=s, out_dtype=out, gelu=gelu)
    oq.oq_check()
    assert torch.equal(s, s_ref)
    assert torch.equal(y.view(torch.int32 if out == torch.float32 else torch.int16),
                       y_ref.view(torch.int32 if out == torch.float32 else torch.int16))
    # and without the norms output (kept internal)
    y2 = oq.oq_quantized_linear(r, ca, cw, x, wc, rn, out_dtype=out, gelu=gelu)
    oq.oq_check()
    assert torch.equal(y2, y)


def test_quantized_linear_back_to_back_on_one_stream(oq):
    """Kernels launched with programmatic stream serialisation start while their predecessor
    finishes and wait for it before touching data.  Steps that follow each other on one
    stream, with x rewritten in place by a torch kernel between them and the pooled workspace
    reused, each equal the two-call result for the x they saw."""
    p = synth.get("flux_attn_w4a4")[0]
    x0 = synth.activations(p, rows=np.arange(0, 1024)).cuda()
    x1 = synth.activations(p, rows=np.arange(1024, 2048)).cuda()
    W = (torch.randn(3072, p.d, generator=torch.Generator().manual_seed(7)) /
         math.sqrt(p.d)).cuda()
    r = oq.oq_build_rpbh(p.d, p.h, 0)
    ca, cw = oq.oq_lloyd_max(p.d, 4), oq.oq_lloyd_max(p.d, 4)
    wc, rn = oq.oq_quantize_weight(r, cw, W)
    refs = []
    for xx in (x0, x1, 2 * x0):
        xc, s = oq.oq_quantize_act(r, ca, xx)
        refs.append(oq.oq_linear(ca, cw, xc, s, wc, rn))
    x = x0.clone()
    ys = []
    for k in range(3):
        if k == 1:
            x.copy_(x1)                                   # a torch kernel between two steps
        if k == 2:
            x.copy_(x0).mul_(2)
        ys.append(oq.oq_quantized_linear(r, ca, cw, x, wc, rn))
    oq.oq_check()
    for y, ref in zip(ys, refs):
        assert torch.equal(y.view(torch.int32), ref.view(torch.int32))


@pytest.mark.parametrize("d,h,ba,bw,T,N", [(256, 64, 4, 4, 64, 256), (3072, 128, 4, 4, 50, 48)])
def test_quantized_linear_fp32_input(oq, d, h, ba, bw, T, N):
    """fp32 x takes the in-call fallback (packed codes, then the decode prepass): y and s are
    still bit-identical to oq_quantize_act + oq_linear, and y is within the linear bound of
    the fp64 oracle on the same codes."""
    g = torch.Generator().manual_seed(d + T)
    x = torch.randn(T, d, generator=g).cuda()
    W = (torch.randn(N, d, generator=g) / math.sqrt(d)).cuda()
    r = oq.oq_build_rpbh(d, h, 0)
    ca, cw = oq.oq_lloyd_max(d, ba), oq.oq_lloyd_max(d, bw)
    wc, rn = oq.oq_quantize_weight(r, cw, W)
    xc, s_ref = oq.oq_quantize_act(r, ca, x)
    y_ref = oq.oq_linear(ca, cw, xc, s_ref, wc, rn)
    s = torch.empty(T, device="cuda")
    y = oq.oq_quantized_linear(r, ca, cw, x, wc, rn, s=s)
    oq.oq_check()
    assert torch.equal(s, s_ref)
    assert torch.equal(y.view(torch.int32), y_ref.view(torch.int32))
    ref = O.linear(xc.cpu().numpy(), s_ref.cpu().double().numpy(), wc.cpu().numpy(),
                   rn.cpu().double().numpy(), d, ba, bw)
    assert rel_l2(y.cpu().double().numpy(), ref) <= LINEAR_RTOL


@pytest.mark.parametrize("h", [2, 4, 8, 16])
@pytest.mark.parametrize("bits,dtype,d,gelu", [
    (4, torch.bfloat16, 1024, False),     # one CTA per SM, named-barrier groups
    (3, torch.float32, 384, False),       # fp32 rows, lockstep groups
    (8, torch.bfloat16, 2560, False),     # bf16 rows, lockstep groups
    (2, torch.bfloat16, 3072, False),
    (4, torch.bfloat16, 1024, True),      # fused GELU
])
def test_k1_blocks_below_32(oq, h, bits, dtype, d, gelu):
    """Hadamard blocks of 2, 4, 8 and 16 (a thread's 32 positions hold several whole blocks):
    codes and norms against the oracle, odd T so the last token pair has one token."""
    T = 45
    p = synth.sweep_projection(d, 128, 4, T)
    x = synth.activations(p)
    if gelu:
        x = (x.float() * torch.exp(torch.randn(T, 1, generator=torch.Generator().manual_seed(h))))
    x = x.to(dtype)
    r = oq.oq_build_rpbh(d, h, 0)
    cb = oq.oq_lloyd_max(d, bits)
    xc, s = oq.oq_quantize_act(r, cb, x.cuda(), gelu=gelu)
    oq.oq_check()
    perm, sign = O.build_rpbh(d, 0)
    o, os_, _, ou = O.quantize_act(x.double().numpy(), h, perm, sign, bits, detail=True,
                                   gelu_input=gelu)
    # GELU sends every strongly negative input to almost zero, and a block of 2 or 4 such
    # values rotates to almost zero, which is the middle boundary of every codebook here: on
    # this input about 0.6 % (h = 2) and 0.1 % (h = 4) of the values lie within 2e-6 sigma of
    # a boundary, far more than the 0.01 % the count rule allows for.  There every mismatch
    # must still be a neighbour code within 1e-5 sigma of their boundary, without the count.
    concentrated = gelu and h <= 4
    check_codes(xc.cpu().numpy(), o, ou, d, bits, f"h={h} b={bits} d={d}",
                count_rule=not concentrated)
    np.testing.assert_allclose(s.cpu().double().numpy(), os_, rtol=NORM_RTOL)


def test_quantized_linear_with_blocks_below_32(oq):
    """h = 8 takes the one-call path's fallback (packed codes, then the decode prepass): y and
    s bit-identical to the two calls, and y within the linear bound of the oracle."""
    d, h, T, N = 1024, 8, 77, 272
    p = synth.sweep_projection(d, 128, 4, T)
    x = synth.activations(p).cuda()
    W = (torch.randn(N, d, generator=torch.Generator().manual_seed(3)) / math.sqrt(d)).cuda()
    r = oq.oq_build_rpbh(d, h, 0)
    ca, cw = oq.oq_lloyd_max(d, 4), oq.oq_lloyd_max(d, 4)
    wc, rn = oq.oq_quantize_weight(r, cw, W)
    xc, s_ref = oq.oq_quantize_act(r, ca, x)
    y_ref = oq.oq_linear(ca, cw, xc, s_ref, wc, rn)
    s = torch.empty(T, device="cuda")
    y = oq.oq_quantized_linear(r, ca, cw, x, wc, rn, s=s)
    oq.oq_check()
    assert torch.equal(s, s_ref)
    assert torch.equal(y.view(torch.int32), y_ref.view(torch.int32))
    ref = O.linear(xc.cpu().numpy(), s_ref.cpu().double().numpy(), wc.cpu().numpy(),
                   rn.cpu().double().numpy(), d, 4, 4)
    assert rel_l2(y.cpu().double().numpy(), ref) <= LINEAR_RTOL


@pytest.mark.parametrize("N,out_dtype", [(20, torch.float32), (4, torch.float32),
                                         (24, torch.bfloat16), (8, torch.bfloat16)])
def test_linear_output_widths_below_16(oq, N, out_dtype):
    """out_features that only satisfy the 16-byte row rule of y (not a multiple of 16): the
    GEMM's last column tile is mostly outside y and its store is clipped.  Against the oracle
    (random codes), and oq_quantized_linear bit-identical to the two calls."""
    T, d, ba, bw = 131, 512, 4, 4
    rng = np.random.default_rng(N)
    xc = O.pack(rng.integers(0, 1 << ba, (T, d)).astype(np.uint8), ba)
    wc = O.pack(rng.integers(0, 1 << bw, (N, d)).astype(np.uint8), bw)
    s = rng.uniform(0.1, 50.0, T)
    rn = rng.uniform(0.5, 2.0, N)
    ca, cw = oq.oq_lloyd_max(d, ba), oq.oq_lloyd_max(d, bw)
    y = oq.oq_linear(ca, cw, torch.from_numpy(xc).cuda(),
                     torch.from_numpy(s.astype(np.float32)).cuda(), torch.from_numpy(wc).cuda(),
                     torch.from_numpy(rn.astype(np.float32)).cuda(), out_dtype=out_dtype)
    oq.oq_check()
    ref = O.linear(xc, s, wc, rn, d, ba, bw)
    tol = LINEAR_RTOL + (BF16_REL if out_dtype == torch.bfloat16 else 0.0)
    assert rel_l2(y.cpu().double().numpy(), ref) <= tol
    p = synth.sweep_projection(d, 128, 4, T)
    x = synth.activations(p).cuda()
    W = (torch.randn(N, d, generator=torch.Generator().manual_seed(N)) / math.sqrt(d)).cuda()
    r = oq.oq_build_rpbh(d, 128, 0)
    wcg, rng_ = oq.oq_quantize_weight(r, cw, W)
    xcg, sg = oq.oq_quantize_act(r, ca, x)
    y2 = oq.oq_linear(ca, cw, xcg, sg, wcg, rng_, out_dtype=out_dtype)
    y1 = oq.oq_quantized_linear(r, ca, cw, x, wcg, rng_, out_dtype=out_dtype)
    oq.oq_check()
    assert torch.equal(y1, y2)
