"""The allocation-free routing call, checked against the regular one.

gnf4_route_permute_static serves callers that may not allocate device
memory (a plugin whose device memory belongs to its host process, or code
that cannot afford cudaMalloc's implicit synchronisation): it keeps its
scratch in a fixed array inside the library.  This file is collected last
so that a failure here never hides the rest of the suite.
"""
import numpy as np
import pytest
import torch

from bit_grouped_moe_b200 import inputs

pytestmark = pytest.mark.gpu


def _alloc(T, k, E, K):
    M = T * k
    mk = lambda n: torch.full((n,), -3, dtype=torch.int32, device="cuda")  # noqa: E731
    return (mk(E + 1), mk(M), mk(M), torch.full((M, K), 5.0, dtype=torch.bfloat16, device="cuda"), mk(1))


def test_static_route_matches_workspace_route_on_two_calls():
    from bit_grouped_moe_b200 import gnf4

    # two calls in a row, both above 256 pairs (the multi-kernel routing that
    # uses the shared array), with different E and chunk counts, so the second
    # call must overwrite the first call's per-chunk histograms
    cases = [(4096, 8, 384, 7168, "zipf"), (300, 4, 128, 64, "uniform")]
    for n, (T, k, E, K, kind) in enumerate(cases):
        rng = inputs.rng(900 + n)
        if kind == "zipf":
            ids, _ = inputs.route_topk(rng, T, k, E, zipf_s=1.2)
        else:
            ids, _ = inputs.route_uniform(rng, T, k, E)
        ids[0, 0] = E  # one dropped pair
        x = torch.from_numpy(inputs.bf16_normal(rng, (T, K)).view(np.int16)).view(torch.bfloat16).cuda()
        d_ids = torch.from_numpy(ids).cuda()
        ref = _alloc(T, k, E, K)
        got = _alloc(T, k, E, K)
        ws = torch.empty(max(gnf4.route_workspace_bytes(T, k, E), 16), dtype=torch.uint8, device="cuda")
        gnf4.route_permute(d_ids, x, E, ref[0], ref[1], ref[2], ref[3], ws, bad_id_count=ref[4])
        gnf4.route_permute_static(d_ids, x, E, got[0], got[1], got[2], got[3], bad_id_count=got[4])
        torch.cuda.synchronize()
        # integer and byte outputs: the tolerance is exact equality
        for a, b in zip(ref[:3] + ref[4:], got[:3] + got[4:]):
            assert torch.equal(a, b)
        assert torch.equal(ref[3].view(torch.int16), got[3].view(torch.int16))
        assert int(got[4].item()) == 1


def test_static_route_refuses_oversized_shapes():
    from bit_grouped_moe_b200 import gnf4

    T, k, E = 1 << 16, 8, 1024  # needs far more scratch than the fixed array holds
    assert gnf4.route_workspace_bytes(T, k, E) > gnf4.ROUTE_STATIC_SCRATCH_BYTES
    st = gnf4._lib.gnf4_route_permute_static(None, None, T, k, E, 64, None, None, None, None, None, None)
    assert st == gnf4.ERR_UNSUPPORTED_SHAPE
    assert "static array" in gnf4.last_error()
