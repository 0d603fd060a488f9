"""The CUDA path against a layer worked by hand, without the oracle.

The layer of tests/golden/hand_moe_layer.json at H = I = 256 (the library's shapes need
multiples of 64, and of 256 for the FP4 tensor cores): two experts with constant weights whose
NVFP4 values are exact (gate/up rows 1.0 / 1.0 for expert 0, 0.5 / 2.0 for expert 1; down
rows 0.25), token 0 = e_0 and token 1 = 2 e_0 - e_1, so sum(x) = 1 for both.  By hand:
h_0 = bf16(silu(1)) = 0.73046875, h_1 = bf16(2 silu(0.5)) = 0.62109375, y_e = 0.25 * 256 * h_e
(46.75 and 39.75), token 0 = 0.75 y_0 + 0.25 y_1 = 45.0 and token 1 = 0.5 y_1 + 0.5 y_0 =
43.25 in every output column, all bf16 values.  Every path must return them bit for bit:
the batched GEMV kernels (two tokens), the one-token GEMV kernels (token 0 alone), the
tcgen05 GEMM path and the FP4 tensor cores (W4A4: the activation rows quantize exactly too).
"""
import json
import os

import pytest
import torch

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
H = I = 256


@pytest.fixture(scope="module")
def nv():
    import bit_quantized_moe_nvfp4_b200 as m
    return m


@pytest.fixture(scope="module")
def hand():
    with open(os.path.join(GOLDEN, "hand_moe_layer.json")) as f:
        g = json.load(f)
    E, T = g["E"], g["T"]
    gu = torch.zeros((E, 2 * I, H), dtype=torch.bfloat16)
    dn = torch.zeros((E, H, I), dtype=torch.bfloat16)
    for e in range(E):
        gu[e, :I] = g["w_gu_gate"][e]
        gu[e, I:] = g["w_gu_up"][e]
        dn[e] = g["w_dn"][e]
    x = torch.zeros((T, H), dtype=torch.bfloat16)
    for t in range(T):
        x[t, :2] = torch.tensor(g["x"][t])
    ids = torch.tensor(g["ids"], dtype=torch.int32)
    w = torch.tensor(g["w"], dtype=torch.float32)
    # y_e = 0.25 * I * h_e, out_t = sum_k w[t, k] * y_ids[t, k]  (the hand working, at I)
    y = [0.25 * I * h for h in g["h"]]
    want = [sum(float(w[t, k]) * y[int(ids[t, k])] for k in range(2)) for t in range(T)]
    assert want == [45.0, 43.25]
    return gu, dn, x, ids, w, torch.tensor(want, dtype=torch.float32)


def _check(out, want):
    o = out.float().cpu()
    assert torch.equal(o, want[:, None].expand_as(o)), o[:, :4]


@pytest.mark.parametrize("path", ["gemv", "gemm"])
def test_hand_layer_two_tokens(nv, hand, path):
    gu, dn, x, ids, w, want = hand
    dev = torch.device("cuda")
    weights = list(nv.nvfp4_quantize(gu.to(dev))) + list(nv.nvfp4_quantize(dn.to(dev)))
    p = nv.PATH_GEMV if path == "gemv" else nv.PATH_GEMM
    out = nv.moe_nvfp4_forward(x.to(dev), ids.to(dev), w.to(dev), *weights, path=p)
    _check(out, want)


def test_hand_layer_one_token(nv, hand):
    gu, dn, x, ids, w, want = hand
    dev = torch.device("cuda")
    weights = list(nv.nvfp4_quantize(gu.to(dev))) + list(nv.nvfp4_quantize(dn.to(dev)))
    out = nv.moe_nvfp4_forward(x[:1].to(dev), ids[:1].to(dev), w[:1].to(dev), *weights,
                               path=nv.PATH_GEMV)
    _check(out, want[:1])


def test_hand_layer_w4a4(nv, hand):
    gu, dn, x, ids, w, want = hand
    dev = torch.device("cuda")
    pg, sg, gg = nv.nvfp4_quantize(gu.to(dev))
    pd, sd, gd = nv.nvfp4_quantize(dn.to(dev))
    sg = nv.nvfp4_w4a4_prepare_scales(sg, gate_rows=I)
    sd = nv.nvfp4_w4a4_prepare_scales(sd)
    out = nv.moe_nvfp4_forward_w4a4(x.to(dev), ids.to(dev), w.to(dev), pg, sg, gg, pd, sd, gd)
    _check(out, want)
