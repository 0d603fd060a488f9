"""The device-side failure path on the GPU, made to happen on purpose without a fault.

Every wait in the library's kernels is bounded by wall-clock time.  The test hook
nvfp4_selftest_wait_timeout runs each kind of wait (an mbarrier phase no thread arrives at,
bulk-copy bytes that never land, a grid-wide counter no CTA advances) with a 2 ms limit and
nothing to complete it: the kernel must return on its own, record bit 1 in the flag, and
leave the context usable, so that the next forward on the same workspace runs, matches the
oracle and clears the flag."""
import time

import pytest
import torch

import synth
from helpers import Layer, compare_moe

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import bit_quantized_moe_nvfp4_b200 as m
    return m


@pytest.mark.parametrize("kind", [0, 1, 2], ids=["mbarrier", "bulk_bytes", "counter"])
def test_wait_gives_up_and_context_survives(nv, kind):
    E, H, I, K, T = 8, 192, 128, 4, 3
    layer = Layer(E, H, I, seed=31)
    x = synth.activations_bf16(T, H, 31)
    ids, w = synth.routing(T, E, K, seed=31)
    ws = nv.alloc_moe_workspace(T, H, I, E, K)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    nv.nvfp4_selftest_wait_timeout(ws, kind, 2_000_000)     # 2 ms
    flag = nv.moe_nvfp4_read_error_flag(ws)                 # synchronises: the kernel ended
    elapsed = time.perf_counter() - t0
    assert flag == 2
    assert elapsed < 1.0
    for path in (nv.PATH_GEMV, nv.PATH_GEMM):
        out = nv.moe_nvfp4_forward(x.cuda(), ids.cuda(), w.cuda(), *layer.dev, workspace=ws,
                                   path=path)
        assert nv.moe_nvfp4_read_error_flag(ws) == 0
        ref, ref64, _ = layer.oracle_forward(x, ids, w)
        compare_moe(out, ref, ref64)
