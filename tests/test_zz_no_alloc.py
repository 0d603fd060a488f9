"""moe_nvfp4_forward_static (fixed library scratch, no workspace) against moe_nvfp4_forward.

Both run the GEMV kernels, so the static call must reproduce the workspace call on the same
inputs; the bar is the MoE tolerance of the parity tests (relative Frobenius error <= 2e-3,
max abs error <= 1e-2 * max|ref|).  Two calls in a row with different batches check that
what the first call leaves in the shared scratch does not leak into the second.  This file
is collected last and needs nothing from the other test files, so it passes alone too."""
import pytest
import torch

import synth
from helpers import MAX_ABS, REL_FRO

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import bit_quantized_moe_nvfp4_b200 as m
    return m


def _layer(nv, E, H, I, seed):
    gu, dn = synth.expert_weights_bf16(E, H, I, seed, device="cuda")
    return list(nv.nvfp4_quantize(gu)) + list(nv.nvfp4_quantize(dn))


def _close(got, ref):
    g, r = got.double(), ref.double()
    nr = torch.linalg.vector_norm(r).item()
    assert nr > 0.0
    rel = (torch.linalg.vector_norm(g - r).item()) / nr
    mab = (g - r).abs().max().item() / r.abs().max().item()
    assert rel <= REL_FRO, f"relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert mab <= MAX_ABS, f"max abs error {mab:.3e} * max|ref| > {MAX_ABS}"


def _batch(T, E, K, H, seed):
    x = synth.activations_bf16(T, H, seed).cuda()
    ids, w = synth.routing(T, E, K, seed, zipf_bias=1.0)
    return x, ids.cuda(), w.cuda()


@pytest.mark.parametrize("shape", [(32, 6144, 2048, 8, [16, 3]), (16, 192, 128, 4, [37, 5]),
                                   (32, 6144, 2048, 8, [1, 1, 1]), (16, 192, 128, 8, [1, 1])],
                         ids=["h6144_i2048", "h192_i128", "h6144_i2048_t1", "h192_i128_t1"])
def test_two_calls_match_workspace_forward(nv, shape):
    E, H, I, K, Ts = shape
    layer = _layer(nv, E, H, I, seed=11)
    flag = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for n, T in enumerate(Ts):
        x, ids, w = _batch(T, E, K, H, seed=100 + n)
        got = nv.moe_nvfp4_forward_static(x, ids, w, *layer, error_flag=flag)
        ref = nv.moe_nvfp4_forward(x, ids, w, *layer, path=nv.PATH_GEMV)
        torch.cuda.synchronize()
        _close(got, ref)
        assert int(flag.item()) == 0


def test_bad_id_sets_flag(nv):
    E, H, I, K, T = 8, 128, 64, 2, 6
    layer = _layer(nv, E, H, I, seed=3)
    x, ids, w = _batch(T, E, K, H, seed=4)
    ids[2, 1] = E + 5
    flag = torch.zeros((1,), dtype=torch.int32, device="cuda")
    got = nv.moe_nvfp4_forward_static(x, ids, w, *layer, error_flag=flag)
    ws = nv.alloc_moe_workspace(T, H, I, E, K)
    ref = nv.moe_nvfp4_forward(x, ids, w, *layer, workspace=ws, path=nv.PATH_GEMV)
    _close(got, ref)
    assert int(flag.item()) == nv.moe_nvfp4_read_error_flag(ws) == 1
    # the next good call clears it
    ids[2, 1] = 0
    nv.moe_nvfp4_forward_static(x, ids, w, *layer, out=got, error_flag=flag)
    assert int(flag.item()) == 0


def test_single_token_bad_id_then_clean_call(nv):
    """One token runs the single-token kernels, which keep their work counters at the start
    of the fixed scratch: a call with an out-of-range id raises the flag, and the clean calls
    after it clear the flag and still match the workspace forward."""
    E, H, I, K = 32, 6144, 2048, 8
    layer = _layer(nv, E, H, I, seed=5)
    flag = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    x, ids, w = _batch(1, E, K, H, seed=6)
    ids_bad = ids.clone()
    ids_bad[0, 3] = -2
    got = nv.moe_nvfp4_forward_static(x, ids_bad, w, *layer, error_flag=flag)
    ws = nv.alloc_moe_workspace(1, H, I, E, K)
    ref = nv.moe_nvfp4_forward(x, ids_bad, w, *layer, workspace=ws, path=nv.PATH_GEMV)
    _close(got, ref)
    assert int(flag.item()) == nv.moe_nvfp4_read_error_flag(ws) == 1
    for n in range(2):
        x, ids, w = _batch(1, E, K, H, seed=7 + n)
        got = nv.moe_nvfp4_forward_static(x, ids, w, *layer, error_flag=flag)
        ref = nv.moe_nvfp4_forward(x, ids, w, *layer, workspace=ws, path=nv.PATH_GEMV)
        torch.cuda.synchronize()
        _close(got, ref)
        assert int(flag.item()) == 0


def test_batch_above_the_fixed_scratch_is_rejected(nv):
    # per pair the scratch holds 2*I + 4*H bytes: 19 tokens x 8 pairs do not fit in 4 MiB
    E, H, I, K, T = 1, 6144, 2048, 8, 19
    dev = "cuda"
    w_gu = torch.zeros((E, 2 * I, H // 2), dtype=torch.uint8, device=dev)
    s_gu = torch.zeros((E, 2 * I, H // 16), dtype=torch.uint8, device=dev)
    w_dn = torch.zeros((E, H, I // 2), dtype=torch.uint8, device=dev)
    s_dn = torch.zeros((E, H, I // 16), dtype=torch.uint8, device=dev)
    g = torch.ones((E,), dtype=torch.float32, device=dev)
    x = torch.zeros((T, H), dtype=torch.bfloat16, device=dev)
    ids = torch.zeros((T, K), dtype=torch.int32, device=dev)
    w = torch.zeros((T, K), dtype=torch.float32, device=dev)
    with pytest.raises(nv.NVFP4Error, match="ESHAPE"):
        nv.moe_nvfp4_forward_static(x, ids, w, w_gu, s_gu, g, w_dn, s_dn, g)
