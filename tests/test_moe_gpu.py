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
from helpers import Layer, compare_moe

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


@pytest.fixture(scope="module")
def full(nv):
    return FullLayer(nv)


def _check_sampled(full, x, ids, w, out, tokens):
    """Compare the listed tokens of `out` with the oracle, token by token, in one oracle call
    over the union of their experts."""
    tokens = sorted(set(int(t) for t in tokens))
    experts = sorted(set(int(e) for t in tokens for e in ids[t]))
    remap = {e: i for i, e in enumerate(experts)}
    ids_s = torch.tensor([[remap[int(e)] for e in ids[t]] for t in tokens], dtype=torch.int32)
    host = full.oracle_inputs(experts)
    ref, ref64, bad = oracle.moe_forward(x[tokens], ids_s, w[tokens], *host)
    assert bad == 0
    for n, t in enumerate(tokens):
        compare_moe(out[t:t + 1], ref[n:n + 1], ref64[n:n + 1])


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


@pytest.mark.parametrize("path", PATHS, ids=["gemv", "gemm"])
@pytest.mark.parametrize("T", [1, 8, 32, 64])
def test_full_layer_decode(nv, full, path, T):
    wl = synth.decode_batch(T)
    x = synth.activations_bf16(T, wl.H, 100 + T)
    ids, w = synth.routing(T, wl.E, wl.K, seed=100 + T)
    out = nv.moe_nvfp4_forward(x.cuda(), ids.cuda(), w.cuda(), *full.dev, path=path)
    torch.cuda.synchronize()
    _check_sampled(full, x, ids, w, out, tokens=[0, T // 2, T - 1])


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
        _check_sampled(full, x, ids, w, out, tokens=[0])


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
    _check_sampled(full, x, ids, w, out, tokens=tokens)
    # the rest of the batch: cheap invariants over every token
    o = out.float()
    assert torch.isfinite(o).all()
    assert (o.abs().amax(dim=1) > 0).all()
