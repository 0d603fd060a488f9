"""Shared helpers for the GPU parity tests: seeded layers, oracle comparison, tolerances.

Tolerance for the MoE forward (bf16 output, fp32 accumulation): relative Frobenius error
<= 2e-3 and max abs error <= 1e-2 * max|ref|, against the oracle's bf16-rounded output.
"""
import numpy as np
import torch

import oracle
import synth

REL_FRO = 2e-3
MAX_ABS = 1e-2


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def compare_moe(out_gpu: torch.Tensor, ref_u16: np.ndarray, ref64: np.ndarray = None):
    """Returns (rel_fro, max_abs_rel) against the bf16 oracle output and asserts the bar."""
    g = out_gpu.detach().float().cpu().numpy().astype(np.float64)
    r = oracle.bf16_bits_to_f32(ref_u16).astype(np.float64).reshape(g.shape)
    nr = np.linalg.norm(r)
    if nr == 0.0:
        assert np.all(g == 0.0)
        return 0.0, 0.0
    rel = float(np.linalg.norm(g - r) / nr)
    mab = float(np.abs(g - r).max() / np.abs(r).max())
    assert rel <= REL_FRO, f"relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert mab <= MAX_ABS, f"max abs error {mab:.3e} * max|ref| > {MAX_ABS}"
    return rel, mab


def compare_partial(part_gpu: torch.Tensor, ref64: np.ndarray):
    """An fp32 partial output (expert-parallel forward) against the oracle's fp64 sum over
    the same pairs; the bar of compare_moe.  An all-zero reference needs an all-zero
    partial."""
    g = part_gpu.detach().cpu().numpy().astype(np.float64)
    r = np.asarray(ref64, np.float64).reshape(g.shape)
    nr = np.linalg.norm(r)
    if nr == 0.0:
        assert np.all(g == 0.0)
        return 0.0, 0.0
    rel = float(np.linalg.norm(g - r) / nr)
    mab = float(np.abs(g - r).max() / np.abs(r).max())
    assert rel <= REL_FRO, f"relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert mab <= MAX_ABS, f"max abs error {mab:.3e} * max|ref| > {MAX_ABS}"
    return rel, mab


def owned_weights(ids: torch.Tensor, w: torch.Tensor, E: int, G: int, r: int) -> torch.Tensor:
    """topk_w with every slot that rank r of G does not serve set to 0: the oracle's
    forward with these weights is rank r's partial (w * y = 0 for the other slots)."""
    own = (ids >= 0) & (ids < E) & (torch.remainder(ids, G) == r)
    return torch.where(own, w, torch.zeros_like(w))


class Layer:
    """A seeded MoE layer: bf16 weights drawn by synth, quantized by the ORACLE on the host
    and copied to the device (small layers only)."""

    def __init__(self, E, H, I, seed=0, std=0.02, outlier_p=0.0, device="cuda"):
        self.E, self.H, self.I = E, H, I
        gu, dn = synth.expert_weights_bf16(E, H, I, seed, std=std, outlier_p=outlier_p)
        self.host = oracle.quantize(gu) + oracle.quantize(dn)   # pg, sg, gg, pd, sd, gd
        self.dev = [torch.from_numpy(np.ascontiguousarray(a)).to(device) for a in self.host]

    def oracle_forward(self, x, ids, w, tokens=None):
        return oracle.moe_forward(x, ids, w, *self.host, tokens=tokens)


class FullLayer:
    """All 256 experts of the H=6144, I=2048 layer on the GPU, quantized by the GPU
    quantizer (N(0, 0.02) bf16 weights).  The oracle's copy of an expert is quantized by
    the oracle from the same seeded bf16 draw, after checking it equals the GPU bytes, and
    kept per expert so that tokens sharing experts reuse it."""

    def __init__(self, nv, seed=0):
        wl = synth.DECODE_T1
        self.E, self.H, self.I, self.seed = wl.E, wl.H, wl.I, seed
        self._cache = {}
        self.dev = []
        for proj, shape in (("w_gu", (2 * self.I, self.H)), ("w_dn", (self.H, self.I))):
            x = torch.empty((self.E,) + shape, dtype=torch.bfloat16, device="cuda")
            for e in range(self.E):
                x[e] = synth.normal_bf16(shape, seed, proj, e, std=0.02, device="cuda")
            self.dev += list(nv.nvfp4_quantize(x))
            del x
        torch.cuda.empty_cache()

    def _expert(self, e):
        if e not in self._cache:
            host = []
            for pi, (proj, shape) in enumerate((("w_gu", (2 * self.I, self.H)),
                                                ("w_dn", (self.H, self.I)))):
                x = synth.normal_bf16(shape, self.seed, proj, e, std=0.02, device="cuda").cpu()
                rp, rs, rg = oracle.quantize(x)
                assert np.array_equal(self.dev[3 * pi][e].cpu().numpy(), rp[0])
                assert np.array_equal(self.dev[3 * pi + 1][e].cpu().numpy(), rs[0])
                assert np.array_equal(self.dev[3 * pi + 2][e:e + 1].cpu().numpy().view(np.uint32),
                                      rg.view(np.uint32))
                host += [rp[0], rs[0], rg[0]]
            self._cache[e] = host
        return self._cache[e]

    def oracle_inputs(self, experts):
        """Oracle-quantized weights of the listed experts, stacked in that order."""
        per = [self._expert(e) for e in experts]
        return [np.stack([p[i] for p in per]) for i in range(6)]


def check_sampled(full, x, ids, w, out, tokens, ep=None, w4a4=False):
    """Compare the listed tokens of `out` with the oracle, token by token, in one oracle call
    over the union of their experts.  ep=(G, r): `out` is rank r's fp32 partial of an
    expert-parallel forward over G ranks, compared with the oracle's sum over that rank's
    slots."""
    tokens = sorted(set(int(t) for t in tokens))
    experts = sorted(set(int(e) for t in tokens for e in ids[t]))
    remap = {e: i for i, e in enumerate(experts)}
    ids_s = torch.tensor([[remap[int(e)] for e in ids[t]] for t in tokens], dtype=torch.int32)
    host = full.oracle_inputs(experts)
    w_s = w[tokens] if ep is None else owned_weights(ids[tokens], w[tokens], full.E, *ep)
    ref, ref64, bad = oracle.moe_forward(x[tokens], ids_s, w_s, *host, w4a4=w4a4)
    assert bad == 0
    for n, t in enumerate(tokens):
        if ep is None:
            compare_moe(out[t:t + 1], ref[n:n + 1], ref64[n:n + 1])
        else:
            compare_partial(out[t:t + 1], ref64[n:n + 1])


def prefill_probe_tokens(ids, tile_n, per_light=6, heavy=4):
    """Tokens of a Zipf-routed batch whose outputs exercise the GEMM path's corner cases:
    a token of each of the `per_light` lightest non-empty experts (a tile with only a few
    occupied slots), the tokens of the first and last slot of the last partial n-tile of
    each of the `heavy` heaviest experts, and one token from each half of the batch."""
    a = ids.numpy()
    T, K = a.shape
    flat = a.reshape(-1)
    counts = np.bincount(flat, minlength=int(flat.max()) + 1)
    nonempty = np.nonzero(counts)[0]
    chosen = []
    for e in nonempty[np.argsort(counts[nonempty], kind="stable")[:per_light]]:
        chosen.append(int(np.nonzero(flat == e)[0][0]) // K)
    for e in np.argsort(-counts, kind="stable")[:heavy]:
        pairs = np.nonzero(flat == e)[0]          # ascending pair index = slot order
        n = pairs.size
        first_of_last_tile = (n - 1) // tile_n * tile_n
        chosen += [int(pairs[first_of_last_tile]) // K, int(pairs[-1]) // K]
    chosen += [0, T // 2 + 1, T - 1]
    return sorted(set(chosen))
