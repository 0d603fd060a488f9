"""Seeded synthetic inputs for the NVFP4 MoE layer.

This module only makes data: bf16 weights and activations drawn from normal laws, router
logits, and routing decisions for the routed-expert tests.  It holds none of the method's
arithmetic (no quantisation, no expert math), so both the CUDA path and the CPU oracle may
take their inputs from it.  routing() turns random logits into (ids, weights) with numpy
and torch in fp64 so that the layer's inputs look like a router's output; the library's
own router is tested only on router_logits() against the oracle's router, never against
routing().

Workloads follow the routed-expert MoE of page "GLM-5-NVFP4-MTP", "Model Description"
(256 experts, 8 active per token) at hidden size 6144 and expert intermediate size 2048:

* weights ~ N(0, 0.02) in bf16, optionally with a Bernoulli(1e-3) fraction of outliers
  scaled by 20;
* activations x ~ N(0, 1) in bf16;
* router logits ~ N(0, 1) per token and expert, optionally plus a Zipf-like bias
  1.5 * ln(1 / (e + 1)) for expert e; routing = softmax -> top-k (ties: lower expert
  index first) -> renormalise, in fp64, weights stored as fp32.

Every draw comes from a ``torch.Generator`` seeded with a value derived from
(seed, stream name), so a tensor can be regenerated piece by piece (one expert at a
time) on any device.  Values differ between CPU and CUDA generators; a workload is
always generated on one device and copied to the other.
"""
from __future__ import annotations

import dataclasses
import hashlib

import numpy as np
import torch


def sub_seed(seed: int, *names) -> int:
    """Stable 63-bit seed for the stream (seed, names...)."""
    h = hashlib.sha256(repr((int(seed),) + tuple(names)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device, seed: int, *names) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(sub_seed(seed, *names))
    return g


def normal_bf16(shape, seed: int, *names, std: float = 1.0, device="cpu",
                outlier_p: float = 0.0, outlier_scale: float = 20.0) -> torch.Tensor:
    """N(0, std^2) drawn in fp32, optionally with outliers, rounded to bf16."""
    g = _gen(device, seed, *names)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        v.mul_(std)
    if outlier_p > 0.0:
        mask = torch.rand(shape, generator=g, device=device) < outlier_p
        v = torch.where(mask, v * outlier_scale, v)
    return v.to(torch.bfloat16)


def expert_weights_bf16(E: int, H: int, I: int, seed: int, device="cpu", std: float = 0.02,
                        outlier_p: float = 0.0, experts=None):
    """Per-expert bf16 weights: gate/up [n, 2I, H] and down [n, H, I] for the listed
    experts (all E when None).  Expert e's tensors depend only on (seed, e)."""
    ids = range(E) if experts is None else list(experts)
    gu = torch.empty((len(ids), 2 * I, H), dtype=torch.bfloat16, device=device)
    dn = torch.empty((len(ids), H, I), dtype=torch.bfloat16, device=device)
    for n, e in enumerate(ids):
        gu[n] = normal_bf16((2 * I, H), seed, "w_gu", int(e), std=std, device=device,
                            outlier_p=outlier_p)
        dn[n] = normal_bf16((H, I), seed, "w_dn", int(e), std=std, device=device,
                            outlier_p=outlier_p)
    return gu, dn


def activations_bf16(T: int, H: int, seed: int, device="cpu") -> torch.Tensor:
    return normal_bf16((T, H), seed, "x", device=device)


def router_logits(T: int, E: int, seed: int, zipf_bias: float = 0.0) -> torch.Tensor:
    """Router logits fp32 [T, E] on the CPU: N(0,1) + zipf_bias * ln(1/(e+1)), rounded to
    fp32 (the same draw as routing() with the same seed)."""
    g = _gen("cpu", seed, "router")
    logits = torch.randn((T, E), generator=g, dtype=torch.float64)
    if zipf_bias:
        e = torch.arange(E, dtype=torch.float64)
        logits = logits + zipf_bias * torch.log(1.0 / (e + 1.0))
    return logits.float()


def routing(T: int, E: int, K: int, seed: int, zipf_bias: float = 0.0):
    """Router decisions for T tokens: (ids int32 [T,K], w fp32 [T,K]) on the CPU.

    logits[t, e] = N(0,1) + zipf_bias * ln(1/(e+1)); p = softmax(logits);
    ids = the K largest p (stable: lower index first on ties), w = p[ids] / sum p[ids].
    """
    g = _gen("cpu", seed, "router")
    logits = torch.randn((T, E), generator=g, dtype=torch.float64)
    if zipf_bias:
        e = torch.arange(E, dtype=torch.float64)
        logits = logits + zipf_bias * torch.log(1.0 / (e + 1.0))
    p = torch.softmax(logits, dim=-1).numpy()
    order = np.argsort(-p, axis=1, kind="stable")[:, :K]
    top = np.take_along_axis(p, order, axis=1)
    w = top / top.sum(axis=1, keepdims=True)
    return (torch.from_numpy(order.astype(np.int32)),
            torch.from_numpy(w.astype(np.float32)))


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic MoE-layer workload."""
    name: str
    T: int
    H: int
    I: int
    E: int
    K: int
    seed: int = 0
    zipf_bias: float = 0.0
    outlier_p: float = 0.0


# The workloads the tests and the benchmark use (sizes of the layer described above).
TINY = Workload("tiny: H=256 I=128 E=8 top-2 T=4", T=4, H=256, I=128, E=8, K=2)
DECODE_T1 = Workload("decode: H=6144 I=2048 E=256 top-8 T=1", T=1, H=6144, I=2048, E=256, K=8)


def decode_batch(T: int) -> Workload:
    return Workload(f"decode: H=6144 I=2048 E=256 top-8 T={T}", T=T, H=6144, I=2048, E=256, K=8)


PREFILL_T4096 = Workload("prefill: H=6144 I=2048 E=256 top-8 T=4096, Zipf routing",
                         T=4096, H=6144, I=2048, E=256, K=8, zipf_bias=1.5)
CODEC_LAYER = Workload("codec: 256 experts x (gate/up [4096,6144] + down [6144,2048]), "
                       "N(0,0.02) with 0.1% x20 outliers",
                       T=0, H=6144, I=2048, E=256, K=8, outlier_p=1e-3)
