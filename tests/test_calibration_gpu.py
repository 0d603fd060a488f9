"""Calibrated (static) global scales on the GPU against the CPU oracle, bit for bit.

Page "GLM-5-NVFP4-MTP", "Calibration dataset": several calibration passes merged by
element-wise max.  nvfp4_amax measures (and merges) per-tensor amax; nvfp4_quantize_with_amax
quantizes with a given amax in place of the tensor's own."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from test_codec_gpu import near_midpoint_input

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def nv():
    import bit_quantized_moe_nvfp4_b200 as m
    return m


def _same_f32(a, b):
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    return np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.mark.parametrize("shape", [(1, 1, 32), (5, 3, 64), (7, 33, 96), (3, 512, 1024),
                                   (300, 1, 32)])
def test_amax_matches_oracle(nv, shape):
    x = synth.normal_bf16(shape, sum(shape), "amax", std=0.5, outlier_p=0.01)
    if shape[0] > 2:
        x[1] = 0.0
    got = nv.nvfp4_amax(x.cuda())
    assert _same_f32(got.cpu().numpy(), oracle.amax(x))


def test_amax_merge_over_passes(nv):
    """Three passes of different data merged on the GPU by element-wise max equal the
    oracle's merge; a larger running value is kept."""
    xs = [synth.normal_bf16((6, 40, 64), 40 + i, "pass", std=0.5 * (i + 1)) for i in range(3)]
    acc_g = nv.nvfp4_amax(xs[0].cuda())
    acc_o = oracle.amax(xs[0])
    for x in xs[1:]:
        nv.nvfp4_amax(x.cuda(), out=acc_g, merge=True)
        oracle.amax(x, out=acc_o, merge=True)
    assert _same_f32(acc_g.cpu().numpy(), acc_o)
    big = torch.full((6,), 1e4, dtype=torch.float32, device="cuda")
    nv.nvfp4_amax(xs[0].cuda(), out=big, merge=True)
    assert torch.all(big == 1e4)


def _check_with_amax(nv, x, am):
    p, s, g = nv.nvfp4_quantize_with_amax(x.cuda(), torch.from_numpy(am).cuda())
    rp, rs, rg = oracle.quantize_with_amax(x, am)
    torch.cuda.synchronize()
    assert _same_f32(g.cpu().numpy(), rg)
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(p.cpu().numpy(), rp)


def test_calibrated_hand_block(nv):
    gold = json.load(open(os.path.join(GOLDEN, "calibrated_block.json")))
    x = torch.tensor(gold["x"]).to(torch.bfloat16).view(1, 1, 32)
    _check_with_amax(nv, x, np.array([gold["amax"]], np.float32))


@pytest.mark.parametrize("factor", [0.25, 1.0, 3.0])
def test_calibrated_quantize_matches_oracle(nv, factor):
    """Calibrated amax below, at and above the data's own: saturated and in-range blocks."""
    x = synth.normal_bf16((9, 24, 96), 61, "calq", std=1.0, outlier_p=0.02)
    x[4] = 0.0
    am = oracle.amax(x) * np.float32(factor)
    am[7] = 0.0                       # an amax of 0 means g = 1
    _check_with_amax(nv, x, am)


def test_calibrated_quantize_near_midpoints(nv):
    x = near_midpoint_input()
    _check_with_amax(nv, x, oracle.amax(x) * np.float32(0.9))
    _check_with_amax(nv, x, oracle.amax(x))


def test_two_pass_quantize_equals_quantize(nv):
    """amax then quantize-with-amax on the same data gives nvfp4_quantize's bytes."""
    x = synth.normal_bf16((4, 256, 512), 71, "twopass", std=0.02, outlier_p=1e-3).cuda()
    a = nv.nvfp4_quantize(x)
    b = nv.nvfp4_quantize_with_amax(x, nv.nvfp4_amax(x))
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_calibrated_layer_sampled(nv):
    """Sixteen gate/up experts of the codec layer quantized with an amax merged over two
    calibration passes (the weights, and the weights scaled by 1.5); three experts drawn
    from the seed are checked bit for bit against the oracle."""
    wl = synth.CODEC_LAYER
    n = 16
    x = torch.empty((n, 2 * wl.I, wl.H), dtype=torch.bfloat16, device="cuda")
    for e in range(n):
        x[e] = synth.normal_bf16((2 * wl.I, wl.H), wl.seed, "w_gu", e, std=0.02, device="cuda",
                                 outlier_p=wl.outlier_p)
    am = nv.nvfp4_amax(x)
    nv.nvfp4_amax((x.float() * 1.5).to(torch.bfloat16), out=am, merge=True)
    p, s, g = nv.nvfp4_quantize_with_amax(x, am)
    torch.cuda.synchronize()
    rng = np.random.default_rng(synth.sub_seed(wl.seed, "calibrated check"))
    for e in sorted(int(v) for v in rng.choice(n, 3, replace=False)):
        xe = x[e:e + 1].cpu()
        ae = oracle.amax(xe)
        oracle.amax((xe.float() * 1.5).to(torch.bfloat16), out=ae, merge=True)
        assert _same_f32(am[e:e + 1].cpu().numpy(), ae)
        rp, rs, rg = oracle.quantize_with_amax(xe, ae)
        assert _same_f32(g[e:e + 1].cpu().numpy(), rg)
        assert np.array_equal(s[e:e + 1].cpu().numpy(), rs)
        assert np.array_equal(p[e:e + 1].cpu().numpy(), rp)
