"""Token permutation on the GPU against the oracle: bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,K,E", [(1, 8, 256), (4, 2, 8), (127, 8, 256), (128, 8, 256),
                                   (129, 8, 256), (4096, 8, 256), (50, 3, 1), (33, 16, 1000),
                                   (3, 8, 1024)])
def test_route_matches_oracle(T, K, E):
    import bit_quantized_moe_nvfp4_b200 as nv
    ids, _ = synth.routing(T, max(E, K), K, seed=T * 31 + K)
    ids = ids.numpy() % E
    if T > 2:
        ids[1, 0] = E          # out of range
        ids[2, K - 1] = -5     # out of range
    counts, offsets, perm, inv, flag = nv.moe_nvfp4_route(torch.from_numpy(ids).cuda(), E)
    rc, ro, rp, ri, bad = oracle.route(ids, E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy()[: ro[E]], rp)
    assert np.array_equal(inv.cpu().numpy(), ri)
    assert int(flag.item()) == (1 if bad else 0)
