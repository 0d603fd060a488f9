"""The BF16 shared expert and the whole layer (router + routed experts + shared expert) on
the GPU against the CPU oracle.

Bar: the layer bar (relative Frobenius <= 2e-3, max abs <= 1e-2 * max|ref| against the
oracle's bf16 output).  The shared expert's h is rounded to bf16 on both sides.  An fp32
sum that lands next to a bf16 rounding boundary can round h the other way, which moves the
output by at most one h ulp times a weight.  That is far inside the bar.
Page "GLM-5-NVFP4-MTP", "What's quantized" (the shared experts stay BF16)."""
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


def shared_weights(H, Is, seed):
    return (synth.normal_bf16((2 * Is, H), seed, "shared_gu", std=0.02),
            synth.normal_bf16((H, Is), seed, "shared_dn", std=0.02))


def reference(x, gu, dn, routed64=None, tokens=None):
    y = oracle.shared_expert(x, gu, dn, tokens=tokens)
    tot = y if routed64 is None else y + routed64
    return oracle.bf16_round_array(tot), tot


# T <= 8: CUDA-core kernels; above: tcgen05 tiles of 256 tokens (ragged last tile), and
# H = 192 / 320 leave a partial 128-row tile in the down projection
@pytest.mark.parametrize("T", [1, 2, 3, 8, 9, 40, 256, 300, 600])
@pytest.mark.parametrize("H,Is", [(192, 128), (320, 256)])
def test_shared_expert_matches_oracle(nv, T, H, Is):
    gu, dn = shared_weights(H, Is, seed=T + H)
    x = synth.activations_bf16(T, H, T + H)
    out = nv.moe_nvfp4_shared_expert(x.cuda(), gu.cuda(), dn.cuda())
    torch.cuda.synchronize()
    ref, ref64 = reference(x, gu, dn)
    compare_moe(out, ref, ref64)


@pytest.mark.parametrize("T", [1, 8, 300])
def test_shared_expert_adds_the_routed_sum(nv, T):
    H, Is = 256, 128
    gu, dn = shared_weights(H, Is, seed=7)
    x = synth.activations_bf16(T, H, 7)
    routed = torch.randn(T, H, generator=torch.Generator().manual_seed(T)) * 0.05
    out = nv.moe_nvfp4_shared_expert(x.cuda(), gu.cuda(), dn.cuda(), routed=routed.cuda())
    torch.cuda.synchronize()
    ref, ref64 = reference(x, gu, dn, routed.double().numpy())
    compare_moe(out, ref, ref64)


def test_shared_expert_zero_tokens_give_the_routed_sum(nv):
    """x = 0: h = 0, so out is the routed sum rounded once to bf16, bit for bit."""
    H, Is = 192, 128
    gu, dn = shared_weights(H, Is, seed=2)
    for T in (4, 20):
        routed = torch.randn(T, H, generator=torch.Generator().manual_seed(T))
        out = nv.moe_nvfp4_shared_expert(torch.zeros(T, H, dtype=torch.bfloat16).cuda(),
                                         gu.cuda(), dn.cuda(), routed=routed.cuda())
        assert torch.equal(out.cpu().view(torch.int16),
                           routed.to(torch.bfloat16).view(torch.int16))


@pytest.mark.parametrize("path", [1, 2], ids=["gemv", "gemm"])
@pytest.mark.parametrize("T", [1, 6, 150])
def test_layer_matches_oracle(nv, path, T):
    E, H, I, K, Is = 16, 192, 128, 4, 128
    layer = Layer(E, H, I, seed=60 + T)
    gu, dn = shared_weights(H, Is, seed=60 + T)
    x = synth.activations_bf16(T, H, 60 + T)
    logits = synth.router_logits(T, E, seed=60 + T, zipf_bias=1.5)
    ids_out = torch.empty((T, K), dtype=torch.int32, device="cuda")
    out = nv.moe_nvfp4_layer(x.cuda(), logits.cuda(), K, *layer.dev, gu.cuda(), dn.cuda(),
                             ids_out=ids_out, path=path)
    torch.cuda.synchronize()
    rid, rw = oracle.router(logits, K)
    assert np.array_equal(ids_out.cpu().numpy(), rid)
    _, routed64, _ = layer.oracle_forward(x, torch.from_numpy(rid),
                                          torch.from_numpy(rw.astype(np.float32)))
    ref, ref64 = reference(x, gu, dn, routed64)
    compare_moe(out, ref, ref64)


@pytest.mark.parametrize("T", [1, 8, 64, 4096])
def test_full_size_shared_expert(nv, T):
    """H = 6144, Is = 2048 (the routed experts' intermediate size), sampled tokens."""
    H, Is = 6144, 2048
    gu = synth.normal_bf16((2 * Is, H), 1, "shared_gu", std=0.02, device="cuda")
    dn = synth.normal_bf16((H, Is), 1, "shared_dn", std=0.02, device="cuda")
    x = synth.activations_bf16(T, H, 90 + T)
    routed = torch.randn(T, H, generator=torch.Generator().manual_seed(5)) * 0.1
    out = nv.moe_nvfp4_shared_expert(x.cuda(), gu, dn, routed=routed.cuda())
    torch.cuda.synchronize()
    tokens = sorted({0, T // 2, T - 1, min(T - 1, 255), min(T - 1, 256)})
    ref, ref64 = reference(x, gu.cpu(), dn.cpu(), routed[tokens].double().numpy(), tokens)
    compare_moe(out[tokens], ref, ref64)
