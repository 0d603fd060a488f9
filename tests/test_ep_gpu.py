"""Expert-parallel forward on one GPU, against the CPU oracle.

The ranks of an expert-parallel group run here one after another on the same device:
every rank is a plain forward over its own experts, and no kernel waits on another rank.
Rank r of G owns the experts e with e % G == r, stored at local index e // G.
  * each rank's fp32 partial is compared with the oracle's sum over that rank's slots
    (the oracle's forward with the other slots' weights set to 0);
  * moe_nvfp4_ep_reduce over the ranks' partials is compared with the oracle's layer
    output, at the bar of the one-GPU forward;
  * with one rank, the reduced partial equals moe_nvfp4_forward's output bit for bit
    (same kernels, same summation order, one rounding);
  * moe_nvfp4_ep_reduce itself is compared bit for bit with a plain fp32 sum in list
    order on the host.
Page "GLM-5-NVFP4-MTP", "How to Run" (multi-GPU serving); "Model Description" (the layer).
"""
import pytest
import torch

import synth
from helpers import (Layer, check_sampled, compare_moe, compare_partial,
                     owned_weights, prefill_probe_tokens)

pytestmark = pytest.mark.gpu

PATHS = [1, 2]   # GEMV, GEMM


@pytest.fixture(scope="module")
def nv():
    import bit_quantized_moe_nvfp4_b200 as m
    return m


def shard(dev, G, r):
    return [t[r::G].contiguous() for t in dev]


def ep_partials(nv, layer_dev, E, x, ids, w, G, path):
    xd, idd, wd = x.cuda(), ids.cuda(), w.cuda()
    parts = []
    for r in range(G):
        parts.append(nv.moe_nvfp4_forward_ep(xd, idd, wd, E, G, r, *shard(layer_dev, G, r),
                                             path=path))
    torch.cuda.synchronize()
    return parts


def test_local_expert_counts(nv):
    for E in (1, 7, 16, 256):
        for G in range(1, min(E, 9) + 1):
            counts = [nv.moe_nvfp4_ep_local_experts(E, G, r) for r in range(G)]
            assert counts == [len(range(r, E, G)) for r in range(G)]
            assert sum(counts) == E
    assert nv.moe_nvfp4_ep_local_experts(8, 3, 3) == 0
    assert nv.moe_nvfp4_ep_local_experts(8, 0, 0) == 0


@pytest.mark.parametrize("path", PATHS, ids=["gemv", "gemm"])
@pytest.mark.parametrize("G", [1, 2, 3, 4])
@pytest.mark.parametrize("T", [1, 5, 37, 200])
def test_small_layer_partials_and_reduction(nv, path, G, T):
    E, H, I, K = 16, 192, 128, 4
    layer = Layer(E, H, I, seed=T + 7, outlier_p=0.01)
    x = synth.activations_bf16(T, H, T + 7)
    ids, w = synth.routing(T, E, K, seed=T + 7, zipf_bias=1.5)
    parts = ep_partials(nv, layer.dev, E, x, ids, w, G, path)
    for r in range(G):
        _, ref64, bad = layer.oracle_forward(x, ids, owned_weights(ids, w, E, G, r))
        assert bad == 0
        compare_partial(parts[r], ref64)
    out = nv.moe_nvfp4_ep_reduce(parts)
    ref, ref64, _ = layer.oracle_forward(x, ids, w)
    compare_moe(out, ref, ref64)
    if G == 1:
        one = nv.moe_nvfp4_forward(x.cuda(), ids.cuda(), w.cuda(), *layer.dev, path=path)
        assert torch.equal(out.view(torch.int16), one.view(torch.int16))


@pytest.mark.parametrize("path", PATHS, ids=["gemv", "gemm"])
def test_foreign_and_bad_ids(nv, path):
    """Slots of another rank's experts are skipped without error; ids outside [0, E) are
    skipped and raise the error flag on every rank; a rank with no slot at all returns
    zeros."""
    E, H, I, K, G, T = 8, 128, 64, 2, 2, 6
    layer = Layer(E, H, I, seed=3)
    x = synth.activations_bf16(T, H, 3)
    ids = torch.tensor([[0, 2], [4, 6], [1, 3], [0, 1], [-1, 2], [E, 5]], dtype=torch.int32)
    w = torch.full((T, K), 0.5, dtype=torch.float32)
    for r in range(G):
        ws = nv.alloc_moe_workspace(T, H, I, nv.moe_nvfp4_ep_local_experts(E, G, r), K)
        part = nv.moe_nvfp4_forward_ep(x.cuda(), ids.cuda(), w.cuda(), E, G, r,
                                       *shard(layer.dev, G, r), workspace=ws, path=path)
        assert nv.moe_nvfp4_read_error_flag(ws) == 1
        _, ref64, _ = layer.oracle_forward(x, ids, owned_weights(ids, w, E, G, r))
        compare_partial(part, ref64)
        # valid ids only: no flag; rank 1 owns none of the even experts
        even = torch.tensor([[0, 2], [4, 6], [2, 0]], dtype=torch.int32)
        part = nv.moe_nvfp4_forward_ep(x[:3].cuda(), even.cuda(), w[:3].cuda(), E, G, r,
                                       *shard(layer.dev, G, r), workspace=ws, path=path)
        assert nv.moe_nvfp4_read_error_flag(ws) == 0
        if r == 1:
            assert torch.all(part == 0)
        else:
            _, ref64, _ = layer.oracle_forward(x[:3], even, w[:3])
            compare_partial(part, ref64)


@pytest.mark.parametrize("n", [1, 2, 3, 8, 16])
@pytest.mark.parametrize("rows,cols", [(1, 4), (37, 192), (300, 6144)])
def test_ep_reduce_is_the_ordered_fp32_sum(nv, n, rows, cols):
    g = torch.Generator().manual_seed(n * 1000 + rows)
    parts = [torch.randn(rows, cols, generator=g) * (10.0 ** (j % 5 - 2)) for j in range(n)]
    parts[0][0, 0] = -0.0
    if n > 1:
        parts[1][0, 1:3] = torch.tensor([3.0, -3.0])
        parts[0][0, 1:3] = torch.tensor([-3.0, 3.0])   # exact cancellation to +0
    want = parts[0].clone()
    for p in parts[1:]:
        want = want + p
    want = want.to(torch.bfloat16)
    got = nv.moe_nvfp4_ep_reduce([p.cuda() for p in parts]).cpu()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_ep_reduce_rejects_bad_arguments(nv):
    p = torch.zeros(4, 8, device="cuda")
    with pytest.raises(ValueError):
        nv.moe_nvfp4_ep_reduce([])
    with pytest.raises(nv.NVFP4Error):
        nv.moe_nvfp4_ep_reduce([p] * (nv.EP_MAX_PARTS + 1))
    with pytest.raises(nv.NVFP4Error):
        nv.moe_nvfp4_ep_reduce([torch.zeros(4, 6, device="cuda")])   # cols % 4


# ----------------------------------------------------------------------------- full size
@pytest.fixture(scope="module")
def full(full_layer):
    return full_layer


@pytest.mark.parametrize("path", PATHS, ids=["gemv", "gemm"])
@pytest.mark.parametrize("T,G", [(1, 8), (8, 2), (64, 4)])
def test_full_layer_decode(nv, full, path, T, G):
    x = synth.activations_bf16(T, full.H, 500 + T)
    ids, w = synth.routing(T, full.E, 8, seed=500 + T)
    parts = ep_partials(nv, full.dev, full.E, x, ids, w, G, path)
    tokens = [0, T // 2, T - 1]
    for r in range(G):
        check_sampled(full, x, ids, w, parts[r], tokens, ep=(G, r))
    check_sampled(full, x, ids, w, nv.moe_nvfp4_ep_reduce(parts), tokens)


@pytest.mark.parametrize("G", [2, 8])
def test_full_layer_prefill(nv, full, G):
    wl = synth.PREFILL_T4096
    x = synth.activations_bf16(wl.T, wl.H, wl.seed + 1)
    ids, w = synth.routing(wl.T, wl.E, wl.K, seed=wl.seed + 1, zipf_bias=wl.zipf_bias)
    parts = ep_partials(nv, full.dev, full.E, x, ids, w, G, path=2)
    out = nv.moe_nvfp4_ep_reduce(parts)
    torch.cuda.synchronize()
    tokens = sorted(set(prefill_probe_tokens(ids, 192)))
    assert len(tokens) >= 8
    for r in (0, G - 1):
        check_sampled(full, x, ids, w, parts[r], tokens, ep=(G, r))
    check_sampled(full, x, ids, w, out, tokens)
    # every token: the reduction of the ranks equals the sum of the partials rounded once
    s = parts[0].clone()
    for p in parts[1:]:
        s += p
    assert torch.equal(out.view(torch.int16), s.to(torch.bfloat16).view(torch.int16))
