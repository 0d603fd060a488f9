"""Pins for the CPU oracle: it is checked against what the format definitions, the
mathematics and independent library routines fix, never against itself.

Format sources: page "GLM-5-NVFP4-MTP", "Model Description" (NVFP4 = 4-bit values with
one FP8 scale per 16 elements; 256 experts, 8 active) and "What's quantized" (routed
expert gate/up/down only).  E2M1 elements, E4M3 scales, one fp32 global scale per tensor
and block scale = amax/6 rounded to E4M3 complete the definition.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# E2M1 codes 0..15 by the bit-field definition (sign | 2-bit exponent, bias 1 | 1-bit
# mantissa; exponent 0 is subnormal), written out value by value.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
              -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def e4m3_torch(codes):
    """E4M3 values through torch's float8_e4m3fn (an independent decoder)."""
    c = torch.as_tensor(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return c.to(torch.float64).numpy()


# ------------------------------------------------------------------------------ E2M1
def test_e2m1_table_exhaustive():
    for code, want in enumerate(E2M1_TABLE):
        got = oracle.e2m1_value(code)
        assert got == want and np.signbit(got) == np.signbit(want), (code, got, want)


@pytest.mark.parametrize("v,code", [
    (0.0, 0x0), (-0.0, 0x8), (0.1, 0x0), (-0.1, 0x8),
    (0.25, 0x0), (0.2500001, 0x1), (0.75, 0x2), (0.7499999, 0x1),
    (1.25, 0x2), (1.2500001, 0x3), (1.75, 0x4), (2.5, 0x4), (2.5000002, 0x5),
    (3.5, 0x6), (3.4999998, 0x5), (5.0, 0x6), (5.0000005, 0x7), (6.0, 0x7),
    (6.5, 0x7), (1e30, 0x7), (-1e30, 0xF), (-2.75, 0xD), (-0.3, 0x9), (4.9, 0x6),
])
def test_e2m1_encode_ties_and_saturation(v, code):
    # Ties go to the even code (mantissa bit 0); above 6 saturates; sign kept on zero.
    assert oracle.e2m1_encode(v) == code


def test_e2m1_encode_roundtrip_every_code():
    for code, val in enumerate(E2M1_TABLE):
        assert oracle.e2m1_encode(val) == code


# ------------------------------------------------------------------------------ E4M3
def test_e4m3_every_code_matches_torch_float8():
    ref = e4m3_torch(np.arange(256))
    for code in range(256):
        got = oracle.e4m3_value(code)
        if np.isnan(ref[code]):
            assert np.isnan(got) and (code & 0x7F) == 0x7F
        else:
            assert got == ref[code], (code, got, ref[code])


def test_e4m3_spot_values():
    assert oracle.e4m3_value(0x7E) == 448.0          # largest finite
    assert oracle.e4m3_value(0x08) == 2.0 ** -6      # smallest normal
    assert oracle.e4m3_value(0x01) == 2.0 ** -9      # smallest subnormal
    assert oracle.e4m3_value(0x07) == 7 * 2.0 ** -9  # largest subnormal
    assert oracle.e4m3_value(0x38) == 1.0
    assert oracle.e4m3_value(0x55) == 13.0


def test_e4m3_monotone_and_roundtrip():
    vals = [oracle.e4m3_value(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))
    for c in range(0x7F):
        assert oracle.e4m3_encode(vals[c]) == c


def test_e4m3_encode_matches_torch_rne():
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.uniform(0, 464, 4000), np.exp(rng.uniform(np.log(1e-4), np.log(448), 4000)),
        rng.uniform(0, 2.0 ** -6, 1000)]).astype(np.float32)
    # midpoints between neighbouring codes: ties to even
    vals = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    v = np.concatenate([v, mids, np.float32(448.0) + np.float32(15.9)[None]])
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(x) for x in v], np.uint8)
    assert np.array_equal(got, want)


def test_e4m3_saturates_instead_of_nan():
    for v in (448.0, 463.9, 464.0, 500.0, 1e6, 3e38):
        assert oracle.e4m3_encode(v) == 0x7E


# ------------------------------------------------------------------------------ bf16
def test_bf16_round_matches_torch_from_fp32():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(20000) * 10 ** rng.uniform(-30, 30, 20000),
                        [0.0, -0.0, 1.0, -3.0]]).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_round(float(x)) for x in v], np.uint16)
    assert np.array_equal(got, want)


def test_bf16_round_is_single_rounding_from_fp64():
    # 1 + 2^-8 is the midpoint between bf16 1.0 and 1 + 2^-7.  A value just above it
    # must round up; rounding through fp32 first would land on the midpoint and go even.
    assert oracle.bf16_round(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    assert oracle.bf16_round(1.0 + 2.0 ** -8) == 0x3F80            # tie -> even
    assert oracle.bf16_round(1.0 + 3 * 2.0 ** -8) == 0x3F82        # tie -> even (up)


# ------------------------------------------------------------------------------ codec
def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)


def test_hand_worked_blocks():
    """Two 16-element blocks worked by hand (tests/golden/hand_block.json)."""
    with open(os.path.join(GOLDEN, "hand_block.json")) as f:
        gold = json.load(f)
    x = _bf16_bits(gold["x"]).reshape(1, 1, 32)
    assert torch.equal(x.float().reshape(-1), torch.tensor(gold["x"]))  # exact in bf16
    packed, scales, g = oracle.quantize(x)
    assert g[0] == np.float32(gold["g"])
    assert list(scales.reshape(-1)) == gold["scales"]
    assert list(packed.reshape(-1)) == [int(b, 16) for b in gold["packed_hex"]]
    deq = oracle.dequantize(packed, scales, g)
    want = _bf16_bits(gold["dequant"]).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(deq.reshape(-1), want)


def _decode_with_tables(packed, scales, g):
    """fp64 weights from packed codes, using the written-out E2M1 table and torch's E4M3."""
    lo = packed & 0xF
    hi = packed >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(*packed.shape[:-1], packed.shape[-1] * 2)
    q = np.asarray(E2M1_TABLE)[codes]
    s = np.repeat(e4m3_torch(scales), 16, axis=-1)
    return q * s * np.asarray(g, np.float64).reshape(-1, *([1] * (packed.ndim - 1)))


def test_quantize_invariants_random():
    x = synth.normal_bf16((3, 24, 96), 7, "inv", std=0.02, outlier_p=0.01)
    x[1, 5, 16:32] = 0.0                      # an all-zero block
    x[2] = 0.0                                # an all-zero tensor
    packed, scales, g = oracle.quantize(x)
    xf = x.double().numpy()
    # zero block and zero tensor
    assert scales[1, 5, 1] == 0 and np.all(packed[1, 5, 8:16] == 0)
    assert g[2] == 1.0 and np.all(scales[2] == 0) and np.all(packed[2] == 0)
    for t in range(2):
        # the block holding the tensor's largest magnitude gets the top scale 448
        amax = np.abs(xf[t]).max()
        assert np.float32(g[t]) == np.float32(np.float32(amax) / np.float32(2688.0))
        r, c = np.unravel_index(np.abs(xf[t]).argmax(), xf[t].shape)
        assert scales[t, r, c // 16] == 0x7E
        # every scale is finite (no NaN code) and no element exceeds 6 * scale * g
        assert np.all((scales[t] & 0x7F) != 0x7F)
    w = _decode_with_tables(packed, scales, g)
    sd = np.repeat(e4m3_torch(scales), 16, axis=-1) * np.asarray(g, np.float64)[:, None, None]
    assert np.all(np.abs(w) <= 6 * sd)
    # reconstruction error is at most one E2M1 grid step of the block (spacing <= 2)
    nz = sd > 0
    assert np.all(np.abs(xf - w)[nz] <= sd[nz] * 1.0 + 1e-12)


def test_dequantize_equals_rounded_exact_product():
    x = synth.normal_bf16((2, 16, 64), 3, "deq", std=0.5)
    packed, scales, g = oracle.quantize(x)
    deq = oracle.dequantize(packed, scales, g)
    # independent: exact product q*s in fp64 -> times g in fp32 -> bf16 via torch
    lo, hi = packed & 0xF, packed >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(2, 16, 64)
    qs = (np.asarray(E2M1_TABLE)[codes] * np.repeat(e4m3_torch(scales), 16, -1)).astype(np.float32)
    v = qs * np.asarray(g, np.float32)[:, None, None]
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(deq, want)


# ------------------------------------------------------------------------------ routing
def test_route_matches_stable_sort():
    ids, _ = synth.routing(37, 16, 4, seed=5)
    ids = ids.numpy().copy()
    ids[3, 1] = 16     # out of range
    ids[7, 0] = -1     # out of range
    ids[9, 2] = ids[9, 3]  # repeated expert within a token
    counts, offsets, perm, inv, bad = oracle.route(ids, 16)
    flat = ids.reshape(-1)
    valid = (flat >= 0) & (flat < 16)
    assert bad == 2
    assert np.array_equal(counts, np.bincount(flat[valid], minlength=16))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    order = np.argsort(np.where(valid, flat, 1 << 20), kind="stable")[: valid.sum()]
    assert np.array_equal(perm, order)
    assert np.all(inv[~valid] == -1)
    assert np.array_equal(perm[inv[valid]], np.nonzero(valid)[0])


# ------------------------------------------------------------------------------ MoE
def _tiny_layer(seed=0, E=8, H=256, I=128):
    gu, dn = synth.expert_weights_bf16(E, H, I, seed)
    pg, sg, gg = oracle.quantize(gu)
    pd, sd, gd = oracle.quantize(dn)
    return pg, sg, gg, pd, sd, gd


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _bf16_np(v):
    # fp64 -> fp32 -> bf16 (torch); differs from a single rounding only on exact fp32 ties
    return torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).double().numpy()


def test_moe_matches_dense_brute_force_tiny():
    wl = synth.TINY
    pg, sg, gg, pd, sd, gd = _tiny_layer(wl.seed, wl.E, wl.H, wl.I)
    x = synth.activations_bf16(wl.T, wl.H, wl.seed)
    ids, w = synth.routing(wl.T, wl.E, wl.K, wl.seed)
    out, out64, bad = oracle.moe_forward(x, ids, w, pg, sg, gg, pd, sd, gd)
    assert bad == 0
    # dense: every expert on every token, weighted by a zero-filled gate matrix
    Wgu = _decode_with_tables(pg, sg, gg)      # [E, 2I, H]
    Wdn = _decode_with_tables(pd, sd, gd)      # [E, H, I]
    G = np.zeros((wl.T, wl.E))
    for t in range(wl.T):
        for k in range(wl.K):
            G[t, ids[t, k]] += float(w[t, k])
    xf = x.double().numpy()
    a = np.einsum("ejh,th->tej", Wgu, xf)                         # [T, E, 2I]
    h = _bf16_np(_silu(a[..., : wl.I]) * a[..., wl.I:])             # [T, E, I]
    y = np.einsum("enj,tej->ten", Wdn, h)                          # [T, E, H]
    dense = np.einsum("te,ten->tn", G, y)
    np.testing.assert_allclose(out64, dense, rtol=1e-9, atol=1e-12 * np.abs(dense).max())
    want_bits = np.array([[oracle.bf16_round(v) for v in row] for row in out64], np.uint16)
    assert np.array_equal(out, want_bits)


def test_moe_single_expert_is_swiglu_mlp():
    H, I, E = 64, 32, 3
    pg, sg, gg, pd, sd, gd = _tiny_layer(4, E, H, I)
    x = synth.activations_bf16(2, H, 4)
    ids = torch.tensor([[2], [0]], dtype=torch.int32)
    w = torch.ones((2, 1), dtype=torch.float32)
    _, out64, _ = oracle.moe_forward(x, ids, w, pg, sg, gg, pd, sd, gd)
    Wgu = _decode_with_tables(pg, sg, gg)
    Wdn = _decode_with_tables(pd, sd, gd)
    for t, e in ((0, 2), (1, 0)):
        xt = x[t].double().numpy()
        gate, up = Wgu[e][:I] @ xt, Wgu[e][I:] @ xt
        want = Wdn[e] @ _bf16_np(_silu(gate) * up)
        np.testing.assert_allclose(out64[t], want, rtol=1e-10, atol=1e-14)


def test_hand_worked_moe_layer():
    """Two constant-weight experts whose NVFP4 values are exact, so the layer output follows
    by hand (tests/golden/hand_moe_layer.json gives the working): SwiGLU on gate rows then up
    rows, the bf16 rounding of h, the down projection and the weighted top-k sum."""
    with open(os.path.join(GOLDEN, "hand_moe_layer.json")) as f:
        gd_ = json.load(f)
    E, H, I, T = gd_["E"], gd_["H"], gd_["I"], gd_["T"]
    gu = torch.zeros((E, 2 * I, H), dtype=torch.bfloat16)
    dn = torch.zeros((E, H, I), dtype=torch.bfloat16)
    for e in range(E):
        gu[e, :I] = gd_["w_gu_gate"][e]
        gu[e, I:] = gd_["w_gu_up"][e]
        dn[e] = gd_["w_dn"][e]
    x = torch.zeros((T, H), dtype=torch.bfloat16)
    for t in range(T):
        x[t, :2] = torch.tensor(gd_["x"][t])
    ids = torch.tensor(gd_["ids"], dtype=torch.int32)
    w = torch.tensor(gd_["w"], dtype=torch.float32)
    pg, sg, gg = oracle.quantize(gu)
    pd, sd, gdn = oracle.quantize(dn)
    code = gd_["element_code"]
    for e in range(E):
        assert np.all(sg[e][:I] == gd_["gate_scale_codes"][e])
        assert np.all(sg[e][I:] == gd_["up_scale_codes"][e])
        assert np.all(sd[e] == gd_["down_scale_codes"][e])
        assert np.all(pg[e] == code | (code << 4)) and np.all(pd[e] == code | (code << 4))
    want = np.repeat(np.asarray(gd_["out"], np.float64)[:, None], H, axis=1)
    # W4A4 too: x rows (e_0; 2 e_0 - e_1) and the constant h rows quantize exactly to NVFP4
    # (every nonzero element is its block maximum or half of it: codes 7 and 13, scale 448)
    for w4a4 in (False, True):
        out, out64, bad = oracle.moe_forward(x, ids, w, pg, sg, gg, pd, sd, gdn, w4a4=w4a4)
        assert bad == 0
        np.testing.assert_allclose(out64, want, rtol=1e-6, atol=0)   # fp32 g: 2^-24
        assert np.array_equal(oracle.bf16_bits_to_f32(out).astype(np.float64), want)


def test_moe_special_cases():
    H, I, E, K, T = 64, 32, 4, 2, 5
    pg, sg, gg, pd, sd, gd = _tiny_layer(9, E, H, I)
    x = synth.activations_bf16(T, H, 9)
    x[1] = 0.0
    x[3] = x[2]
    ids = torch.tensor([[0, 1], [2, 3], [1, 3], [1, 3], [E, 0]], dtype=torch.int32)
    w = torch.tensor([[0.6, 0.4], [0.5, 0.5], [0.3, 0.7], [0.3, 0.7], [0.9, 0.1]])
    out, out64, bad = oracle.moe_forward(x, ids, w, pg, sg, gg, pd, sd, gd)
    assert np.all(out64[1] == 0.0)                      # x = 0 gives 0
    assert np.array_equal(out[2], out[3])               # identical tokens
    assert bad == 1                                     # id E is out of range ...
    ids1 = torch.tensor([[0]], dtype=torch.int32)       # ... and contributes nothing
    _, ref64, _ = oracle.moe_forward(x[4:5], ids1, torch.tensor([[0.1]]),
                                     pg, sg, gg, pd, sd, gd)
    np.testing.assert_allclose(out64[4], ref64[0], rtol=1e-12, atol=0)
    # swapping the two slots of a token (with their weights) changes nothing but fp64
    # summation order
    ids2 = ids[:, [1, 0]].contiguous()
    w2 = w[:, [1, 0]].contiguous()
    _, out64b, _ = oracle.moe_forward(x, ids2, w2, pg, sg, gg, pd, sd, gd)
    np.testing.assert_allclose(out64b, out64, rtol=1e-12, atol=1e-15)


# ----------------------------------------------------------------------------- calibration
def test_calibrated_hand_block():
    """A hand-worked row quantized with a calibrated amax half the data's own: the block
    scale and the codes saturate (tests/golden/calibrated_block.json gives the working)."""
    gold = json.load(open(os.path.join(GOLDEN, "calibrated_block.json")))
    x = torch.tensor(gold["x"], dtype=torch.float32).to(torch.bfloat16).view(1, 1, 32)
    assert torch.equal(x.float().view(-1), torch.tensor(gold["x"]))
    p, s, g = oracle.quantize_with_amax(x, np.array([gold["amax"]], np.float32))
    assert float(g[0]) == gold["g"]
    assert s.reshape(-1).tolist() == gold["scales"]
    codes = np.stack([p.reshape(-1) & 15, p.reshape(-1) >> 4], axis=1).reshape(-1)
    assert codes.tolist() == gold["codes"]
    assert [f"{b:02x}" for b in p.reshape(-1)] == gold["packed_hex"]
    deq = oracle.bf16_bits_to_f32(oracle.dequantize(p, s, g)).reshape(-1)
    want = np.array(gold["dequant"], np.float32)
    assert np.array_equal(deq, want) and np.array_equal(np.signbit(deq), np.signbit(want))


def _planted(n, rows, cols, peaks, seed):
    """bf16 tensors of values below 0.49 in magnitude, each with one planted maximum."""
    g = torch.Generator().manual_seed(seed)
    x = (torch.rand((n, rows, cols), generator=g) * 0.98 - 0.49).to(torch.bfloat16)
    for t, v in enumerate(peaks):
        i = int(torch.randint(0, rows * cols, (1,), generator=g))
        x.view(n, -1)[t, i] = v
    return x


def test_amax_is_the_planted_maximum():
    peaks = [3.5, -7.25, 0.75, 1024.0]
    x = _planted(4, 9, 48, peaks, 3)
    assert oracle.amax(x).tolist() == [abs(v) for v in peaks]
    assert oracle.amax(torch.zeros((2, 3, 16), dtype=torch.bfloat16)).tolist() == [0.0, 0.0]


def test_amax_merge_is_elementwise_max_over_passes():
    """Three calibration passes merged by element-wise max: the result is each tensor's
    largest planted maximum, whatever the order of the passes; a running value larger than
    a pass's amax is kept."""
    passes = [[2.0, 9.0, 0.5], [9.0, -4.0, 0.75], [-4.0, 2.0, 0.625]]
    xs = [_planted(3, 5, 32, p, 10 + i) for i, p in enumerate(passes)]
    want = np.max(np.abs(np.array(passes)), axis=0).astype(np.float32)
    for order in ([0, 1, 2], [2, 0, 1]):
        acc = oracle.amax(xs[order[0]])
        for i in order[1:]:
            oracle.amax(xs[i], out=acc, merge=True)
        assert acc.tolist() == want.tolist()
    acc = np.array([100.0, 100.0, 100.0], np.float32)
    assert oracle.amax(xs[0], out=acc, merge=True).tolist() == [100.0] * 3


def test_quantize_with_own_amax_is_quantize():
    """Given each tensor's own amax, the calibrated quantizer is the plain one."""
    x = synth.normal_bf16((5, 12, 64), 23, "cal", std=0.02, outlier_p=0.02)
    x[2] = 0.0
    a, b = oracle.quantize_with_amax(x, oracle.amax(x)), oracle.quantize(x)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


@pytest.mark.parametrize("factor", [0.25, 4.0])
def test_calibrated_range_invariants(factor):
    """A calibrated amax below the data's saturates (scales at most 448, codes at most 6,
    |dequantized| <= 6 * 448 * g); one above it leaves every block inside the E4M3 range."""
    x = synth.normal_bf16((3, 16, 64), 29, "cal", std=1.0, outlier_p=0.01)
    am = oracle.amax(x) * np.float32(factor)
    p, s, g = oracle.quantize_with_amax(x, am)
    assert np.array_equal(g, am / np.float32(2688.0))
    assert int(s.max()) <= 0x7E
    deq = oracle.bf16_bits_to_f32(oracle.dequantize(p, s, g)).astype(np.float64)
    bound = 6.0 * 448.0 * g.astype(np.float64)[:, None, None]
    assert np.all(np.abs(deq) <= bound * (1 + 2 ** -8))
    if factor > 1:
        assert int(s.max()) < 0x7E
        xf = x.float().numpy().astype(np.float64)
        # inside the range the dequantized block keeps the data's sign and the error is
        # below one E2M1 step of the block
        scl = np.repeat(np.vectorize(oracle.e4m3_value)(s), 16, axis=2) * g[:, None, None]
        assert np.all(np.abs(deq - xf) <= scl * 2.0 + 1e-30)


# ----------------------------------------------------------------------------- router
# Page "GLM-5-NVFP4-MTP", "Model Description" (8 of 256 experts per token); reading: softmax
# -> K largest (lower index first on ties) -> renormalised over the K.

def test_router_equal_logits_pick_the_lowest_indices():
    ids, w = oracle.router(np.zeros((2, 10), np.float32) + np.float32(0.7), 4)
    assert ids.tolist() == [[0, 1, 2, 3]] * 2
    np.testing.assert_allclose(w, 0.25, rtol=0, atol=1e-15)


def test_router_two_value_closed_form():
    # softmax([0, ln 3]) = [1/4, 3/4]; with K = E nothing is dropped
    ids, w = oracle.router(np.array([[0.0, np.log(3.0)]], np.float32), 2)
    assert ids.tolist() == [[1, 0]]
    l1 = float(np.float32(np.log(3.0)))
    want = np.array([np.exp(l1), 1.0]) / (1.0 + np.exp(l1))
    np.testing.assert_allclose(w[0], want, rtol=1e-15)
    np.testing.assert_allclose(w[0], [0.75, 0.25], rtol=1e-7)


def test_router_hand_example_with_a_tie():
    # logits [1, 3, 2, 3]: experts 1 and 3 tie at the top (1 first), then 2;
    # weights e^3 : e^3 : e^2 renormalised = e/(2e+1), e/(2e+1), 1/(2e+1)
    ids, w = oracle.router(np.array([[1.0, 3.0, 2.0, 3.0]], np.float32), 3)
    assert ids.tolist() == [[1, 3, 2]]
    e = np.e
    np.testing.assert_allclose(w[0], [e / (2 * e + 1), e / (2 * e + 1), 1 / (2 * e + 1)],
                               rtol=1e-14)


def test_router_top1_has_weight_one():
    logits = synth.router_logits(50, 37, seed=4)
    ids, w = oracle.router(logits, 1)
    assert np.array_equal(ids[:, 0], np.argmax(logits.numpy(), axis=1))
    assert np.all(w == 1.0)


def test_router_underflowed_probabilities_keep_the_logit_order():
    # exp(-1000) and below underflow to 0 in fp64: the order still follows the logits
    ids, w = oracle.router(np.array([[0.0, -1000.0, -2000.0, -1500.0]], np.float32), 3)
    assert ids.tolist() == [[0, 1, 3]]
    assert w.tolist() == [[1.0, 0.0, 0.0]]


def test_router_shift_invariant():
    logits = synth.router_logits(20, 64, seed=9, zipf_bias=1.5)
    ids0, w0 = oracle.router(logits, 8)
    ids1, w1 = oracle.router(logits + 8.0, 8)   # exact: |logits| < 8, shifts of 8 keep order
    assert np.array_equal(ids0, ids1)
    np.testing.assert_allclose(w0, w1, rtol=1e-5)


def test_router_matches_stable_argsort_and_topk_softmax():
    """Brute force by another route: numpy's stable argsort of -logits for the choice, and
    the softmax of the K chosen logits alone for the weights (the full denominator cancels
    in the renormalisation)."""
    for T, E, K, bias in ((64, 8, 2, 0.0), (33, 256, 8, 1.5), (5, 1024, 16, 0.0)):
        logits = synth.router_logits(T, E, seed=E + K, zipf_bias=bias).numpy()
        ids, w = oracle.router(logits, K)
        want = np.argsort(-logits, axis=1, kind="stable")[:, :K]
        assert np.array_equal(ids, want)
        top = np.take_along_axis(logits.astype(np.float64), want, axis=1)
        ex = np.exp(top - top[:, :1])
        np.testing.assert_allclose(w, ex / ex.sum(axis=1, keepdims=True), rtol=1e-12)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-14)


# ----------------------------------------------------------------------------- shared expert
# Page "GLM-5-NVFP4-MTP", "What's quantized": every weight but the routed experts' stays
# BF16; the shared expert is a dense SwiGLU MLP added to the routed sum.

def test_shared_expert_identity_weights():
    """Gate = identity, up = 2 x identity, down = identity: y_n = bf16(silu(x_n) * 2 x_n).
    Exchanging gate and up would give silu(2 x) * x instead."""
    H = Is = 64
    eye = torch.eye(H, dtype=torch.float32)
    w_gu = torch.cat([eye, 2 * eye]).to(torch.bfloat16)
    w_dn = eye.to(torch.bfloat16)
    x = torch.linspace(-4, 4, H).view(1, H).to(torch.bfloat16)
    y = oracle.shared_expert(x, w_gu, w_dn)
    xv = x.double().numpy()[0]
    want = oracle.bf16_bits_to_f32(oracle.bf16_round_array(xv / (1 + np.exp(-xv)) * 2 * xv))
    np.testing.assert_array_equal(y[0], want.astype(np.float64))
    swapped = 2 * xv / (1 + np.exp(-2 * xv)) * xv
    assert np.abs(y[0] - swapped).max() > 0.1


def test_shared_expert_matches_dense_brute_force():
    T, H, Is = 5, 128, 64
    x = synth.activations_bf16(T, H, 3)
    w_gu = synth.normal_bf16((2 * Is, H), 3, "sgu", std=0.05)
    w_dn = synth.normal_bf16((H, Is), 3, "sdn", std=0.05)
    y = oracle.shared_expert(x, w_gu, w_dn)
    X, G, D = (t.double().numpy() for t in (x, w_gu, w_dn))
    a = X @ G.T
    hh = a[:, :Is] / (1 + np.exp(-a[:, :Is])) * a[:, Is:]
    h = oracle.bf16_bits_to_f32(oracle.bf16_round_array(hh)).astype(np.float64)
    np.testing.assert_allclose(y, h @ D.T, rtol=1e-12, atol=1e-12)
    # a subset of tokens gives the same rows
    np.testing.assert_array_equal(oracle.shared_expert(x, w_gu, w_dn, tokens=[4, 1]), y[[4, 1]])


def test_shared_expert_zero_input_and_down_linearity():
    H, Is = 64, 128
    w_gu = synth.normal_bf16((2 * Is, H), 5, "sgu", std=0.05)
    w_dn = synth.normal_bf16((H, Is), 5, "sdn", std=0.05)
    assert np.all(oracle.shared_expert(torch.zeros(2, H, dtype=torch.bfloat16), w_gu, w_dn) == 0)
    x = synth.activations_bf16(3, H, 5)
    y1 = oracle.shared_expert(x, w_gu, w_dn)
    y2 = oracle.shared_expert(x, w_gu, (w_dn.float() * 2).to(torch.bfloat16))
    np.testing.assert_array_equal(y2, 2 * y1)


def test_bf16_round_array_matches_scalar_rounding():
    v = np.concatenate([synth.router_logits(4, 64, seed=1).double().numpy().ravel() * 1e3,
                        [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -9, 65504.0]])
    assert [int(b) for b in oracle.bf16_round_array(v)] == [oracle.bf16_round(x) for x in v]


# ----------------------------------------------------------------------------- W4A4
# The layer with NVFP4 activations (reading: each x row and each h row quantized as a tensor
# of its own), as the block-scaled FP4 tensor-core GEMM computes it.

def _exact_nvfp4(packed, scales, g):
    """Exact fp64 values of NVFP4 tensors [n, rows, cols/2] + [n, rows, cols/16] + [n]."""
    e2m1 = np.array([oracle.e2m1_value(c) for c in range(16)])
    e4m3 = np.array([oracle.e4m3_value(c) if (c & 0x7F) != 0x7F else 0.0 for c in range(256)])
    lo, hi = packed & 15, packed >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(packed.shape[:-1] + (packed.shape[-1] * 2,))
    sc = np.repeat(e4m3[scales], 16, axis=-1)
    return e2m1[codes] * sc * np.asarray(g, np.float64).reshape((-1,) + (1,) * (packed.ndim - 1))


def test_w4a4_matches_composition_of_pinned_steps():
    """Recompose the W4A4 layer from the pinned quantizer, the exact E2M1/E4M3 tables and the
    pinned bf16 rounding with numpy dense products: quantize each x row, contract with the
    exact weights, SwiGLU, round h to bf16, quantize each h row, contract, combine."""
    E, H, I, K, T = 6, 64, 32, 2, 5
    gu, dn = synth.expert_weights_bf16(E, H, I, seed=8, outlier_p=0.02)
    pg, sg, gg = oracle.quantize(gu)
    pd, sd, gd = oracle.quantize(dn)
    Wg, Wd = _exact_nvfp4(pg, sg, gg), _exact_nvfp4(pd, sd, gd)
    x = synth.activations_bf16(T, H, 8)
    ids, w = synth.routing(T, E, K, seed=8)
    _, out64, bad = oracle.moe_forward(x, ids, w, pg, sg, gg, pd, sd, gd, w4a4=True)
    assert bad == 0
    want = np.zeros((T, H))
    for t in range(T):
        qp, qs, qg = oracle.quantize(x[t:t + 1].view(1, 1, H))
        xq = _exact_nvfp4(qp, qs, qg)[0, 0]
        for k in range(K):
            e = int(ids[t, k])
            a = Wg[e] @ xq
            hh = a[:I] / (1 + np.exp(-a[:I])) * a[I:]
            hb = torch.from_numpy(oracle.bf16_round_array(hh).astype(np.int16)).view(
                torch.bfloat16).view(1, 1, I)
            hp, hs, hg = oracle.quantize(hb)
            want[t] += float(w[t, k]) * (Wd[e] @ _exact_nvfp4(hp, hs, hg)[0, 0])
    np.testing.assert_allclose(out64, want, rtol=1e-11, atol=1e-13)


def test_w4a4_special_cases():
    E, H, I, K, T = 4, 64, 32, 2, 3
    gu, dn = synth.expert_weights_bf16(E, H, I, seed=9)
    wts = oracle.quantize(gu) + oracle.quantize(dn)
    ids, w = synth.routing(T, E, K, seed=9)
    out, out64, _ = oracle.moe_forward(torch.zeros(T, H, dtype=torch.bfloat16), ids, w, *wts,
                                       w4a4=True)
    assert np.all(out64 == 0)
    # quantizing activations moves the output by the NVFP4 noise of x and h, not more
    x = synth.activations_bf16(T, H, 9)
    _, a16, _ = oracle.moe_forward(x, ids, w, *wts)
    _, a4, _ = oracle.moe_forward(x, ids, w, *wts, w4a4=True)
    rel = np.linalg.norm(a4 - a16) / np.linalg.norm(a16)
    assert 1e-3 < rel < 0.25
