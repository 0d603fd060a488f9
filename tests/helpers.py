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
