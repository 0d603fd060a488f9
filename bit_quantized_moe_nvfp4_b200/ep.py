"""Expert parallelism: one process per GPU, the routed experts split across the ranks.

Page "GLM-5-NVFP4-MTP", "How to Run", serves the model on several GPUs at once with NCCL
between them.  The routed-expert layer splits by expert.  Rank r of G owns the experts e
with e % G == r and keeps them at local index e // G, which spreads a Zipf-skewed routing
evenly.  Every rank holds the same tokens and routing and computes, with the library's
kernels (moe_nvfp4_forward_ep), the fp32 partial sum over its own (token, slot) pairs.
The one exchange step sums the partials over the ranks with an NCCL collective, through
torch.distributed:
  * "all_reduce": every rank receives all T rows of the layer output;
  * "reduce_scatter": rank r receives rows [r*T/G, (r+1)*T/G) (T a multiple of G). This
    moves about half the bytes, for callers whose next step is sharded by token.
moe_nvfp4_ep_reduce then rounds the summed rows to bf16 on each rank.  The rounding
happens once, after the sum over all experts, as in the one-GPU forward.

This module holds only the host-side plumbing: the partition, the collective and the
call order.  All arithmetic runs in the library's kernels and in NCCL.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (PATH_AUTO, moe_nvfp4_ep_local_experts, moe_nvfp4_ep_reduce,
               moe_nvfp4_forward_ep)

MODES = ("all_reduce", "reduce_scatter")


def local_experts(E: int, ep_size: int, ep_rank: int) -> list[int]:
    """Global ids of the experts rank ep_rank owns, in local-index order."""
    if not (1 <= ep_size <= E and 0 <= ep_rank < ep_size):
        raise ValueError(f"rank {ep_rank} of {ep_size} over {E} experts")
    return list(range(ep_rank, E, ep_size))


def shard_experts(tensors, ep_size: int, ep_rank: int):
    """This rank's slices of per-expert tensors (leading dimension E), contiguous."""
    return [t[ep_rank::ep_size].contiguous() for t in tensors]


def kept_rows(T: int, ep_size: int, ep_rank: int, mode: str) -> slice:
    """Rows of the layer output that rank ep_rank holds after the exchange."""
    if mode == "all_reduce":
        return slice(0, T)
    if mode == "reduce_scatter":
        if T % ep_size:
            raise ValueError(f"reduce_scatter needs T ({T}) to be a multiple of {ep_size}")
        n = T // ep_size
        return slice(ep_rank * n, (ep_rank + 1) * n)
    raise ValueError(f"mode must be one of {MODES}")


def reduce_partial(partial: torch.Tensor, group=None, mode: str = "all_reduce",
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """Sum the fp32 partial [T, H] over the ranks of `group`; return the summed rows
    this rank keeps (kept_rows).  all_reduce sums in place."""
    G, r = dist.get_world_size(group), dist.get_rank(group)
    rows = kept_rows(partial.shape[0], G, r, mode)
    if mode == "all_reduce":
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
        return partial
    if out is None:
        out = partial.new_empty((rows.stop - rows.start,) + tuple(partial.shape[1:]))
    dist.reduce_scatter_tensor(out, partial, op=dist.ReduceOp.SUM, group=group)
    return out


class ExpertParallelMoE:
    """The layer's routed experts on one rank of an expert-parallel group.

    local_weights: (w_gu, s_gu, g_gu, w_dn, s_dn, g_dn) of the experts local_experts()
    names, in that order (shard_experts of the whole layer gives them).  Buffers (the
    partial, the summed rows, the workspace) are allocated once per token count and
    reused, so a step can be captured in a CUDA graph."""

    def __init__(self, E: int, local_weights, group=None, mode: str = "all_reduce",
                 path: int = PATH_AUTO):
        if mode not in MODES:
            raise ValueError(f"mode must be one of {MODES}")
        self.group, self.mode, self.path, self.E = group, mode, path, E
        self.size, self.rank = dist.get_world_size(group), dist.get_rank(group)
        self.weights = tuple(local_weights)
        n_loc = moe_nvfp4_ep_local_experts(E, self.size, self.rank)
        if self.weights[0].shape[0] != n_loc:
            raise ValueError(f"rank {self.rank} of {self.size} owns {n_loc} experts, "
                             f"got {self.weights[0].shape[0]}")
        self._buf = {}

    def _buffers(self, T: int, H: int, K: int, device):
        key = (T, H, K)
        if key not in self._buf:
            from . import alloc_moe_workspace
            I = self.weights[0].shape[1] // 2
            n_loc = self.weights[0].shape[0]
            rows = kept_rows(T, self.size, self.rank, self.mode)
            n = rows.stop - rows.start
            self._buf[key] = (
                torch.empty((T, H), dtype=torch.float32, device=device),
                torch.empty((n, H), dtype=torch.float32, device=device),
                torch.empty((n, H), dtype=torch.bfloat16, device=device),
                alloc_moe_workspace(T, H, I, n_loc, K, device),
            )
        return self._buf[key]

    def forward(self, x, topk_ids, topk_w) -> torch.Tensor:
        """The layer output rows this rank keeps (bf16 [len(kept_rows), H])."""
        T, H = x.shape
        partial, summed, out, ws = self._buffers(T, H, topk_ids.shape[1], x.device)
        moe_nvfp4_forward_ep(x, topk_ids, topk_w, self.E, self.size, self.rank,
                             *self.weights, out=partial, workspace=ws, path=self.path)
        summed = reduce_partial(partial, self.group, self.mode,
                                out=summed if self.mode == "reduce_scatter" else None)
        return moe_nvfp4_ep_reduce([summed], out=out)

    def workspace(self, T: int, H: int, K: int, device):
        """The workspace used for T tokens (its first word is the error flag)."""
        return self._buffers(T, H, K, device)[3]
