"""Expert parallelism's host side on CPU: gloo ranks, one process each, as under torchrun.

Each rank takes its experts with the package's partition (ep.local_experts /
ep.shard_experts), computes its partial with the oracle on those local weights only
(slots of other ranks' experts get weight 0), and the package's exchange step
(ep.reduce_partial, all_reduce or reduce_scatter) sums the partials.  The rows each rank
keeps, rounded to bf16, must match the oracle's output of the whole layer.  A wrong
partition (an expert served twice, or by nobody, or a wrong local index) or a wrong
reduction fails the comparison.  Page "GLM-5-NVFP4-MTP", "How to Run" (multi-GPU serving).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
E, H, I, K, T = 12, 128, 64, 4, 6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer():
    import oracle
    import synth
    gu, dn = synth.expert_weights_bf16(E, H, I, seed=5)
    host = oracle.quantize(gu) + oracle.quantize(dn)
    x = synth.activations_bf16(T, H, 5)
    ids, w = synth.routing(T, E, K, seed=5, zipf_bias=1.5)
    return host, x, ids, w


def _rank_main(rank, world, port, mode, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import oracle
    from bit_quantized_moe_nvfp4_b200 import ep
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        host, x, ids, w = _layer()
        mine = ep.local_experts(E, world, rank)
        local = ep.shard_experts([torch.from_numpy(np.ascontiguousarray(a)) for a in host],
                                 world, rank)
        # ids in local numbering; slots of other ranks' experts: any local id, weight 0
        where = {e: i for i, e in enumerate(mine)}
        ids_l = torch.tensor([[where.get(int(e), 0) for e in row] for row in ids],
                             dtype=torch.int32)
        own = torch.tensor([[int(e) in where for e in row] for row in ids])
        w_l = torch.where(own, w, torch.zeros_like(w))
        _, part64, bad = oracle.moe_forward(x, ids_l, w_l, *[t.numpy() for t in local])
        assert bad == 0
        partial = torch.from_numpy(np.asarray(part64, np.float64).astype(np.float32)).view(T, H)
        summed = ep.reduce_partial(partial.contiguous(), mode=mode)
        rows = ep.kept_rows(T, world, rank, mode)
        out[rank] = (rows.start, rows.stop, summed.to(torch.bfloat16).view(torch.int16).numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", ["all_reduce", "reduce_scatter"])
@pytest.mark.parametrize("world", [2, 3])
def test_partition_and_exchange_match_the_whole_layer(world, mode):
    sys.path.insert(0, ROOT)
    import oracle
    from helpers import compare_moe
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, mode, out), nprocs=world, join=True)
        got = dict(out)
    host, x, ids, w = _layer()
    ref, ref64, _ = oracle.moe_forward(x, ids, w, *host)
    ref = np.asarray(ref).reshape(T, H)
    ref64 = np.asarray(ref64).reshape(T, H)
    covered = []
    for rank in range(world):
        a, b, bits = got[rank]
        covered += list(range(a, b))
        rows = torch.from_numpy(bits).view(torch.bfloat16)
        compare_moe(rows, ref[a:b], ref64[a:b])
    if mode == "all_reduce":
        assert covered == list(range(T)) * world
    else:
        assert covered == list(range(T))


def test_partition_covers_every_expert_once():
    sys.path.insert(0, ROOT)
    from bit_quantized_moe_nvfp4_b200 import ep
    for E_ in (1, 5, 16, 256):
        for G in range(1, min(E_, 8) + 1):
            owned = sorted(e for r in range(G) for e in ep.local_experts(E_, G, r))
            assert owned == list(range(E_))
            for r in range(G):
                assert all(e % G == r for e in ep.local_experts(E_, G, r))
    with pytest.raises(ValueError):
        ep.local_experts(4, 5, 0)
    with pytest.raises(ValueError):
        ep.kept_rows(7, 2, 0, "reduce_scatter")


def test_library_local_count_matches_the_partition():
    """moe_nvfp4_ep_local_experts (C, no CUDA call) against the host partition."""
    sys.path.insert(0, ROOT)
    from bit_quantized_moe_nvfp4_b200 import build, ep
    import bit_quantized_moe_nvfp4_b200 as nv
    build.build()
    for E_ in (1, 7, 256):
        for G in range(1, min(E_, 8) + 1):
            for r in range(G):
                assert nv.moe_nvfp4_ep_local_experts(E_, G, r) == len(ep.local_experts(E_, G, r))
