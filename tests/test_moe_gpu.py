"""MoE forward on the GPU against the CPU oracle (both kernel paths).

Bar: relative Frobenius error <= 2e-3 and max abs error <= 1e-2 * max|ref| against the
oracle's bf16 output (bf16 output, fp32 accumulation).  At full layer size the oracle
computes sampled tokens one by one; the weights it reads are quantized by the oracle from
the same seeded bf16 draws, after checking they equal the GPU quantizer's bytes."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import Layer, check_sampled, compare_moe, prefill_probe_tokens

pytestmark = pytest.mark.gpu

PATHS = [1, 2]   # GEMV (CUDA cores), GEMM (tcgen05)


@pytest.fixture(scope="module")
def nv():
    import bit_quantized_moe_nvfp4_b200 as m
    return m


def run(nv, layer, x, ids, w, path):
    return nv.moe_nvfp4_forward(x.cuda(), ids.cuda(), w.cuda(), *layer.dev, path=path)


@pytest.mark.parametrize("path", PATHS, ids=["gemv", "gemm"])
def test_tiny_layer(nv, path):
    wl = synth.TINY
    layer = Layer(wl.E, wl.H, wl.I, wl.seed)
    x = synth.activations_bf16(wl.T, wl.H, wl.seed)
    ids, w = synth.routing(wl.T, wl.E, wl.K, wl.seed)
    out = run(nv, layer, x, ids, w, path)
    ref, ref64, _ = layer.oracle_forward(x, ids, w)
    compare_moe(out, ref, ref64)


@pytest.mark.parametrize("path", PATHS, ids=["gemv", "gemm"])
@pytest.mark.parametrize("T", [1, 5, 37, 200])
def test_small_layer_many_shapes(nv, path, T):
    E, H, I, K = 16, 192, 128, 4
    layer = Layer(E, H, I, seed=T, outlier_p=0.01)
    x = synth.activations_bf16(T, H, T)
    ids, w = synth.routing(T, E, K, seed=T, zipf_bias=1.5)
    out = run(nv, layer, x, ids, w, path)
    ref, ref64, _ = layer.oracle_forward(x, ids, w)
    compare_moe(out, ref, ref64)


@pytest.mark.parametrize("path", PATHS, ids=["gemv", "gemm"])
def test_batch_sizes_alternating(nv, path):
    """Larger, smaller, then larger batches again on the same kernels: each launch needs
    its own amount of shared memory, and a smaller call must not leave a kernel unable to
    launch a larger one."""
    E, H, I, K = 37, 192, 128, 4
    layer = Layer(E, H, I, seed=21)
    for n, T in enumerate([40, 3, 40, 9]):
        x = synth.activations_bf16(T, H, 50 + n)
        ids, w = synth.routing(T, E, K, seed=50 + n)
        out = run(nv, layer, x, ids, w, path)
        ref, ref64, _ = layer.oracle_forward(x, ids, w)
        compare_moe(out, ref, ref64)


@pytest.mark.parametrize("path", PATHS, ids=["gemv", "gemm"])
def test_edge_cases(nv, path):
    """One expert takes every token, most experts are empty, a zero token, a repeated id
    within a token, and an out-of-range id (contributes nothing, raises the flag)."""
    E, H, I, K, T = 6, 128, 64, 3, 41
    layer = Layer(E, H, I, seed=2)
    x = synth.activations_bf16(T, H, 2)
    x[7] = 0.0
    ids = torch.zeros((T, K), dtype=torch.int32)
    ids[:, 1] = 3
    ids[:, 2] = 3               # repeated id
    ids[5, 2] = E               # out of range
    w = torch.full((T, K), 1.0 / K)
    ws = nv.alloc_moe_workspace(T, H, I, E, K)
    out = nv.moe_nvfp4_forward(x.cuda(), ids.cuda(), w.cuda(), *layer.dev, workspace=ws,
                               path=path)
    assert nv.moe_nvfp4_read_error_flag(ws) & 1
    ref, ref64, bad = layer.oracle_forward(x, ids, w)
    assert bad == 1
    compare_moe(out, ref, ref64)
    assert torch.all(out[7] == 0)
    # a clean call on the same workspace clears the flag
    ids[5, 2] = 1
    nv.moe_nvfp4_forward(x.cuda(), ids.cuda(), w.cuda(), *layer.dev, workspace=ws, path=path)
    assert nv.moe_nvfp4_read_error_flag(ws) == 0


@pytest.mark.parametrize("path", PATHS, ids=["gemv", "gemm"])
def test_single_token_edge_cases(nv, path):
    """One token (the single-token GEMV kernels): an expert picked three times, another
    twice, an out-of-range id, a reduction length that is not a multiple of 128; then a
    token whose ids are all out of range (zero output)."""
    E, H, I, K = 8, 192, 128, 8
    layer = Layer(E, H, I, seed=9)
    x = synth.activations_bf16(1, H, 9)
    ids = torch.tensor([[3, 3, 1, E, 3, 0, 7, 1]], dtype=torch.int32)
    w = torch.arange(1, K + 1, dtype=torch.float32).view(1, K) / 36.0
    ws = nv.alloc_moe_workspace(1, H, I, E, K)
    out = nv.moe_nvfp4_forward(x.cuda(), ids.cuda(), w.cuda(), *layer.dev, workspace=ws,
                               path=path)
    assert nv.moe_nvfp4_read_error_flag(ws) & 1
    ref, ref64, bad = layer.oracle_forward(x, ids, w)
    assert bad == 1
    compare_moe(out, ref, ref64)
    bad_ids = torch.full((1, K), -1, dtype=torch.int32)
    out = nv.moe_nvfp4_forward(x.cuda(), bad_ids.cuda(), w.cuda(), *layer.dev, workspace=ws,
                               path=path)
    assert nv.moe_nvfp4_read_error_flag(ws) & 1
    assert torch.all(out == 0)


# ----------------------------------------------------------------------------- full size
@pytest.fixture(scope="module")
def full(full_layer):
    return full_layer


@pytest.mark.parametrize("path", PATHS, ids=["gemv", "gemm"])
@pytest.mark.parametrize("T", [1, 8, 32, 64])
def test_full_layer_decode(nv, full, path, T):
    wl = synth.decode_batch(T)
    x = synth.activations_bf16(T, wl.H, 100 + T)
    ids, w = synth.routing(T, wl.E, wl.K, seed=100 + T)
    out = nv.moe_nvfp4_forward(x.cuda(), ids.cuda(), w.cuda(), *full.dev, path=path)
    torch.cuda.synchronize()
    check_sampled(full, x, ids, w, out, tokens=[0, T // 2, T - 1])


def test_full_layer_single_token_calls_in_a_row(nv, full):
    """Consecutive one-token calls on one workspace: the gate/up kernel hands out its
    chunks from a counter in the workspace head, which every call must leave at zero for
    the next one; each call is checked against the oracle."""
    wl = synth.DECODE_T1
    ws = nv.alloc_moe_workspace(1, wl.H, wl.I, wl.E, wl.K)
    for n in range(3):
        x = synth.activations_bf16(1, wl.H, 300 + n)
        ids, w = synth.routing(1, wl.E, wl.K, seed=300 + n)
        out = nv.moe_nvfp4_forward(x.cuda(), ids.cuda(), w.cuda(), *full.dev, workspace=ws,
                                   path=1)
        torch.cuda.synchronize()
        assert torch.all(ws[:nv.WORKSPACE_ZERO_BYTES].view(torch.int32)[1:] == 0)
        check_sampled(full, x, ids, w, out, tokens=[0])


@pytest.mark.parametrize("path", [2, 0], ids=["gemm", "auto"])
def test_full_layer_prefill(nv, full, path):
    wl = synth.PREFILL_T4096
    x = synth.activations_bf16(wl.T, wl.H, wl.seed)
    ids, w = synth.routing(wl.T, wl.E, wl.K, seed=wl.seed, zipf_bias=wl.zipf_bias)
    out = nv.moe_nvfp4_forward(x.cuda(), ids.cuda(), w.cuda(), *full.dev, path=path)
    torch.cuda.synchronize()
    # n-tiles of 192 slots (the GEMM path's tile) and of 128 / 256 slots
    tokens = sorted(set(sum((prefill_probe_tokens(ids, n) for n in (128, 192, 256)), [])))
    assert len(tokens) >= 16
    check_sampled(full, x, ids, w, out, tokens=tokens)
    # the rest of the batch: cheap invariants over every token
    o = out.float()
    assert torch.isfinite(o).all()
    assert (o.abs().amax(dim=1) > 0).all()
