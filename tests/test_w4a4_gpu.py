"""The W4A4 layer on the block-scaled FP4 tensor cores, against the oracle's W4A4 mode.

Bar: the layer bar (relative Frobenius <= 2e-3, max abs <= 1e-2 * max|ref| against the
oracle's bf16 output of the W4A4 function).  The activation codes come from the same
quantizer arithmetic on both sides.  The one place the two can part is h: it is summed in
fp32 on the GPU and in fp64 in the oracle before its bf16 rounding and quantization, so a
value next to a bf16 rounding boundary can take the neighbouring code.  That moves one
element of one h row by one E2M1 step, and is rare (about 1e-5 per element).
Page "GLM-5-NVFP4-MTP", "How to Run" (FP4 quantization and FP4 MoE kernels)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import Layer, check_sampled, compare_moe, prefill_probe_tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import bit_quantized_moe_nvfp4_b200 as m
    return m


def atoms_reference(sc: np.ndarray, gate_rows: int) -> np.ndarray:
    """The tensor cores' scale layout written out with numpy index arithmetic: atom (tensor,
    row group, 64-column chunk) of 512 bytes, row r's four scales at 16 (r % 32) + 4 (r / 32);
    gate/up groups take 64 gate rows then the matching 64 up rows."""
    n, rows, c16 = sc.shape
    groups, chunks = rows // 128, c16 // 4
    r = np.arange(128)
    grp = np.arange(groups)[:, None]
    if gate_rows:
        src = np.where(r < 64, 64 * grp + r, gate_rows + 64 * grp + (r - 64))
    else:
        src = 128 * grp + r
    out = np.zeros((n, groups, chunks, 512), np.uint8)
    pos = 16 * (r % 32) + 4 * (r // 32)
    for c in range(chunks):
        for b in range(4):
            out[:, :, c, pos + b] = sc[:, src, 4 * c + b]
    return out.reshape(sc.shape)


@pytest.mark.parametrize("n,rows,cols,gate", [(1, 128, 64, 0), (3, 256, 512, 128),
                                              (2, 384, 192, 0), (256, 4096, 6144, 2048)])
def test_prepare_scales_layout(nv, n, rows, cols, gate):
    g = torch.Generator().manual_seed(rows + cols)
    sc = torch.randint(0, 256, (n, rows, cols // 16), dtype=torch.uint8, generator=g)
    got = nv.nvfp4_w4a4_prepare_scales(sc.cuda(), gate_rows=gate).cpu().numpy()
    assert np.array_equal(got, atoms_reference(sc.numpy(), gate))


def prepared(nv, dev, I):
    w_gu, s_gu, g_gu, w_dn, s_dn, g_dn = dev
    return (w_gu, nv.nvfp4_w4a4_prepare_scales(s_gu, gate_rows=I), g_gu,
            w_dn, nv.nvfp4_w4a4_prepare_scales(s_dn), g_dn)


@pytest.mark.parametrize("T", [1, 5, 37, 200, 600])
def test_small_layer(nv, T):
    E, H, I, K = 16, 512, 256, 4
    layer = Layer(E, H, I, seed=T + 3, outlier_p=0.01)
    x = synth.activations_bf16(T, H, T + 3)
    ids, w = synth.routing(T, E, K, seed=T + 3, zipf_bias=1.5)
    out = nv.moe_nvfp4_forward_w4a4(x.cuda(), ids.cuda(), w.cuda(),
                                    *prepared(nv, layer.dev, I))
    torch.cuda.synchronize()
    ref, ref64, _ = oracle.moe_forward(x, ids, w, *layer.host, w4a4=True)
    compare_moe(out, ref, ref64)


def test_edge_cases(nv):
    """One expert takes every slot (several 128-slot tiles), most experts empty, a zero
    token, a repeated id and an out-of-range id (error flag, contributes nothing)."""
    E, H, I, K, T = 8, 256, 256, 2, 300
    layer = Layer(E, H, I, seed=5)
    x = synth.activations_bf16(T, H, 5)
    x[7] = 0
    ids = torch.full((T, K), 3, dtype=torch.int32)
    ids[::3, 1] = 5
    ids[11] = torch.tensor([6, 6])
    ids[12, 0] = E
    w = torch.full((T, K), 0.5, dtype=torch.float32)
    ws = torch.zeros((nv.moe_nvfp4_w4a4_workspace_size(T, H, I, E, K),), dtype=torch.uint8,
                     device="cuda")
    out = nv.moe_nvfp4_forward_w4a4(x.cuda(), ids.cuda(), w.cuda(), *prepared(nv, layer.dev, I),
                                    workspace=ws)
    assert nv.moe_nvfp4_read_error_flag(ws) & 1
    ref, ref64, bad = oracle.moe_forward(x, ids, w, *layer.host, w4a4=True)
    assert bad == 1
    compare_moe(out, ref, ref64)
    assert torch.all(out[7] == 0)


@pytest.fixture(scope="module")
def full(full_layer):
    return full_layer


@pytest.fixture(scope="module")
def full_prepared(nv, full):
    return prepared(nv, full.dev, full.I)


@pytest.mark.parametrize("T", [8, 64])
def test_full_layer_small_batches(nv, full, full_prepared, T):
    x = synth.activations_bf16(T, full.H, 700 + T)
    ids, w = synth.routing(T, full.E, 8, seed=700 + T)
    out = nv.moe_nvfp4_forward_w4a4(x.cuda(), ids.cuda(), w.cuda(), *full_prepared)
    torch.cuda.synchronize()
    check_sampled(full, x, ids, w, out, [0, T // 2, T - 1], w4a4=True)


def test_full_layer_prefill(nv, full, full_prepared):
    wl = synth.PREFILL_T4096
    x = synth.activations_bf16(wl.T, wl.H, wl.seed + 2)
    ids, w = synth.routing(wl.T, wl.E, wl.K, seed=wl.seed + 2, zipf_bias=wl.zipf_bias)
    out = nv.moe_nvfp4_forward_w4a4(x.cuda(), ids.cuda(), w.cuda(), *full_prepared)
    torch.cuda.synchronize()
    tokens = sorted(set(prefill_probe_tokens(ids, 128)))
    assert len(tokens) >= 8
    check_sampled(full, x, ids, w, out, tokens, w4a4=True)
    o = out.float()
    assert torch.isfinite(o).all() and (o.abs().amax(dim=1) > 0).all()
