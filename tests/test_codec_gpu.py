"""NVFP4 quantize / dequantize on the GPU against the CPU oracle: bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import bit_quantized_moe_nvfp4_b200 as m
    return m


def _check_quant(nv, x):
    packed, scales, g = nv.nvfp4_quantize(x.cuda())
    rp, rs, rg = oracle.quantize(x.cpu())
    torch.cuda.synchronize()
    assert np.array_equal(g.cpu().numpy().view(np.uint32), rg.view(np.uint32))
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(packed.cpu().numpy(), rp)
    deq = nv.nvfp4_dequantize(packed, scales, g)
    rd = oracle.dequantize(rp, rs, rg)
    assert np.array_equal(deq.cpu().contiguous().view(torch.int16).numpy().view(np.uint16), rd)


def test_tiny_layer_weights(nv):
    wl = synth.TINY
    gu, dn = synth.expert_weights_bf16(wl.E, wl.H, wl.I, wl.seed)
    _check_quant(nv, gu)
    _check_quant(nv, dn)


@pytest.mark.parametrize("shape", [(1, 1, 32), (3, 7, 96), (2, 33, 160), (5, 1, 2048),
                                   (1, 300, 64), (7, 13, 32)])
def test_random_shapes_with_outliers(nv, shape):
    x = synth.normal_bf16(shape, sum(shape), "codec", std=0.02, outlier_p=0.01)
    _check_quant(nv, x)


def test_special_blocks(nv):
    x = synth.normal_bf16((4, 16, 128), 11, "special", std=1.0)
    x[0] = 0.0                                    # all-zero tensor -> g = 1
    x[1, 3, :32] = 0.0                            # zero blocks
    x[1, 4, :16] = -0.0                           # negative zeros
    x[2, 0, 0] = 3.0e4                            # a huge outlier: tiny blocks get
    x[2, 1:, :] *= 1e-4                           # subnormal or zero scales
    x[3, 5, 16:32] = torch.tensor([1e-30] * 16)   # far below the tensor scale
    x[3, 6, :16] = torch.linspace(-6, 6, 16)      # a spread of grid values
    _check_quant(nv, x)


def _near_midpoint_tensor(rows, t_amax, rng):
    """bf16 rows of 32 elements (two 16-element blocks) whose element quotients x / d lie on,
    or within a few fp32 ulps of, an E2M1 rounding midpoint (0.25, 0.75, ..., 5), where the
    search finds such values.  Element 0 fixes the tensor amax (hence g); element 0 of each
    block fixes the block's d (computed with the oracle's own steps); the other 15 come from
    an exhaustive search over the positive bf16 values, with random signs (random values
    where the search finds nothing)."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    allv = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)   # positive bf16
    g = np.float32(np.float32(t_amax) / np.float32(2688.0))
    x = np.zeros((rows, 32), np.float32)
    x[0, 0] = t_amax
    for r in range(1, rows):
        for blk in range(2):
            b_amax = allv[rng.integers(0x3C00, 0x4400)]           # a block amax below t_amax
            sv = np.float32(np.float32(b_amax / np.float32(6.0)) / g)
            s8 = oracle.e4m3_encode(float(sv))
            d = np.float32(np.float32(oracle.e4m3_value(s8)) * g)
            with np.errstate(over="ignore", divide="ignore"):
                q = (allv / d).astype(np.float32)
            near = np.zeros(allv.shape, bool)
            for m in mids:
                near |= np.abs(q - m) <= 4 * np.spacing(m)
            cand = allv[near & (allv <= b_amax)]
            if cand.size == 0:
                cand = allv[(allv <= b_amax) & (allv > b_amax / 64)]
            sign = np.where(rng.random(15) < 0.5, -1.0, 1.0).astype(np.float32)
            x[r, 16 * blk] = b_amax
            x[r, 16 * blk + 1:16 * blk + 16] = rng.choice(cand, 15) * sign
    return x


def near_midpoint_input(rows=48, seed=17):
    """Four tensors: global scales 1 and 0.75 (exact midpoint quotients: ties) and two
    irregular ones (quotients next to a midpoint, where any exist)."""
    rng = np.random.default_rng(seed)
    ts = [_near_midpoint_tensor(rows, a, rng) for a in (2688.0, 2016.0, 1999.0, 2944.0)]
    return torch.from_numpy(np.stack(ts)).to(torch.bfloat16)   # exact: all bf16 values


def test_quantize_near_rounding_midpoints(nv):
    """Element quotients on and next to every E2M1 rounding midpoint: the codes must be those
    of dividing each element by its block's d (the quantizer's fast path defers to IEEE
    division exactly there)."""
    _check_quant(nv, near_midpoint_input())


def test_dequantize_arbitrary_codes(nv):
    g = torch.Generator().manual_seed(3)
    packed = torch.randint(0, 256, (3, 20, 64), generator=g, dtype=torch.uint8)
    scales = torch.randint(0, 256, (3, 20, 8), generator=g, dtype=torch.uint8)
    scales[(scales & 0x7F) == 0x7F] = 0x3C        # no NaN scale codes
    gs = torch.tensor([1.0, 3.7e-3, 2.0 ** -20], dtype=torch.float32)
    deq = nv.nvfp4_dequantize(packed.cuda(), scales.cuda(), gs.cuda())
    rd = oracle.dequantize(packed.numpy(), scales.numpy(), gs.numpy())
    assert np.array_equal(deq.cpu().view(torch.int16).numpy().view(np.uint16), rd)


def _neighbours(v):
    v = np.asarray(v, np.float32)
    return np.concatenate([v, np.nextafter(v, np.float32(np.inf)),
                           np.nextafter(v, np.float32(-np.inf))])


def test_scalar_casts_sweep(nv):
    """Every rounding threshold of both formats, its fp32 neighbours, and random values."""
    e4 = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    mids = (e4[:-1] + e4[1:]) / 2
    e2 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    e2mids = (e2[:-1] + e2[1:]) / 2
    rng = np.random.default_rng(5)
    v = np.concatenate([
        _neighbours(e4), _neighbours(mids), _neighbours(e2), _neighbours(e2mids),
        _neighbours([448.0, 464.0, 500.0, 6.0, 7.0, 1e30, 2.0 ** -9, 2.0 ** -10, 2.0 ** -126]),
        rng.standard_normal(5000) * 10 ** rng.uniform(-12, 4, 5000)]).astype(np.float32)
    v = np.concatenate([v, -v, [0.0, -0.0]]).astype(np.float32)
    g4, g2 = nv.nvfp4_cast_f32(torch.from_numpy(v).cuda())
    want4 = np.array([oracle.e4m3_encode(x) for x in v], np.uint8)
    want2 = np.array([oracle.e2m1_encode(x) for x in v], np.uint8)
    got4, got2 = g4.cpu().numpy(), g2.cpu().numpy()
    bad4 = np.nonzero(got4 != want4)[0]
    bad2 = np.nonzero(got2 != want2)[0]
    assert bad4.size == 0, [(float(v[i]), int(got4[i]), int(want4[i])) for i in bad4[:8]]
    assert bad2.size == 0, [(float(v[i]), int(got2[i]), int(want2[i])) for i in bad2[:8]]


def test_full_layer_codec_sampled(nv):
    """All 256 experts of one layer (gate/up [4096,6144] + down [6144,2048], N(0,0.02)
    with 0.1% x20 outliers), quantized and dequantized in one call per projection on the
    GPU; five experts (the first, the last and three drawn from the seed) are checked bit
    for bit against the oracle."""
    wl = synth.CODEC_LAYER
    E, H, I = wl.E, wl.H, wl.I
    out = {}
    for proj, shape in (("w_gu", (2 * I, H)), ("w_dn", (H, I))):
        x = torch.empty((E,) + shape, dtype=torch.bfloat16, device="cuda")
        for e in range(E):
            x[e] = synth.normal_bf16(shape, wl.seed, proj, e, std=0.02, device="cuda",
                                     outlier_p=wl.outlier_p)
        packed, scales, g = nv.nvfp4_quantize(x)
        deq = nv.nvfp4_dequantize(packed, scales, g)
        torch.cuda.synchronize()
        # the first and last expert, and three drawn from the workload's seed
        rng = np.random.default_rng(synth.sub_seed(wl.seed, "codec check", proj))
        picks = sorted(set([0, E - 1] + [int(v) for v in rng.choice(E, 3, replace=False)]))
        for e in picks:
            rp, rs, rg = oracle.quantize(x[e].cpu())
            assert np.array_equal(g[e:e + 1].cpu().numpy().view(np.uint32), rg.view(np.uint32))
            assert np.array_equal(scales[e].cpu().numpy(), rs[0]), (proj, e)
            assert np.array_equal(packed[e].cpu().numpy(), rp[0]), (proj, e)
            if e == picks[len(picks) // 2]:
                rd = oracle.dequantize(rp, rs, rg)[0]
                got = deq[e].cpu().view(torch.int16).numpy().view(np.uint16)
                assert np.array_equal(got, rd), (proj, e)
        out[proj] = float(g.max())
        del x, packed, scales, g, deq
        torch.cuda.empty_cache()
