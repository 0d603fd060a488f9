"""The router on the GPU against the oracle's router, and the layer run from router logits.

Selection (which experts, in which slot) is compared bit for bit: both sides decide it on
the same fp32 logits.  The fp32 weights are compared with the oracle's fp64 weights at
rtol 4e-6 / atol 1e-7.  That bound comes from the arithmetic: l_k - l_max rounds to half an
fp32 ulp of a value of at most ~20, which is about 1e-6 of relative error after exp.  expf
adds 2 ulp, and the K-term sum and the division add a few more ulps.
Page "GLM-5-NVFP4-MTP", "Model Description" (8 of 256 experts per token)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import Layer, compare_moe

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import bit_quantized_moe_nvfp4_b200 as m
    return m


def check(nv, logits, K):
    ids, w = nv.moe_nvfp4_router(logits.cuda(), K)
    torch.cuda.synchronize()
    rid, rw = oracle.router(logits, K)
    assert np.array_equal(ids.cpu().numpy(), rid)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=4e-6, atol=1e-7)


@pytest.mark.parametrize("T,E,K,bias", [
    (1, 256, 8, 0.0), (7, 256, 8, 1.5), (4096, 256, 8, 1.5), (64, 8, 2, 0.0),
    (33, 37, 5, 0.0), (100, 1024, 16, 1.5), (3, 33, 1, 0.0), (5, 16, 16, 0.0),
    (9, 513, 7, 0.0)])
def test_router_matches_oracle(nv, T, E, K, bias):
    check(nv, synth.router_logits(T, E, seed=T * 31 + E, zipf_bias=bias), K)


def test_router_ties_and_plateaus(nv):
    """Logits on a coarse grid (many equal values across lanes and registers), all-equal
    rows, and rows whose top values repeat: the lower index must win every tie."""
    g = torch.Generator().manual_seed(3)
    coarse = torch.round(torch.randn(200, 256, generator=g) * 2.0) / 2.0
    coarse[0] = 0.25
    coarse[1, ::3] = 5.0
    check(nv, coarse.float(), 8)
    check(nv, coarse[:, :40].contiguous().float(), 16)


def test_router_extreme_spreads(nv):
    """Weights that underflow in fp32 next to the top one, and large logits."""
    logits = torch.tensor([[0.0, -200.0, -90.0, -300.0, 5.0, 80.0, 79.5, -1e4],
                           [1e4, 1e4 - 1.0, -1e4, 3.0, 2.0, 1.0, 0.0, 1e4]], dtype=torch.float32)
    check(nv, logits, 4)


@pytest.mark.parametrize("path", [1, 2], ids=["gemv", "gemm"])
@pytest.mark.parametrize("T", [1, 6, 150])
def test_layer_from_logits(nv, path, T):
    E, H, I, K = 16, 192, 128, 4
    layer = Layer(E, H, I, seed=40 + T)
    x = synth.activations_bf16(T, H, 40 + T)
    logits = synth.router_logits(T, E, seed=40 + T, zipf_bias=1.5)
    ids_out = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w_out = torch.empty((T, K), dtype=torch.float32, device="cuda")
    out = nv.moe_nvfp4_forward_logits(x.cuda(), logits.cuda(), K, *layer.dev, ids_out=ids_out,
                                      w_out=w_out, path=path)
    torch.cuda.synchronize()
    rid, rw = oracle.router(logits, K)
    assert np.array_equal(ids_out.cpu().numpy(), rid)
    np.testing.assert_allclose(w_out.cpu().numpy(), rw, rtol=4e-6, atol=1e-7)
    ref, ref64, _ = layer.oracle_forward(x, torch.from_numpy(rid),
                                         torch.from_numpy(rw.astype(np.float32)))
    compare_moe(out, ref, ref64)
    # without output pointers the decisions stay in the workspace: same layer output
    again = nv.moe_nvfp4_forward_logits(x.cuda(), logits.cuda(), K, *layer.dev, path=path)
    assert torch.equal(again.view(torch.int16), out.view(torch.int16))
