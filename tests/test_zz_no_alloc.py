"""hata_topk_noalloc: top-k for callers that cannot allocate device memory.

Such a caller gets no workspace; the entry point keeps its scratch in a fixed
array owned by the library.  The GPU test checks, through the C ABI, that two
calls in a row give exactly the indices and counts of hata_topk with a
workspace.  This file sorts last so that a run stopping at its first failure
has already run every other test; it also passes on its own in a fresh
process (the first call on the device does the scratch set-up).
"""
import ctypes

import numpy as np
import pytest

from hata_inputs import random_scores


@pytest.fixture(scope="module")
def H():
    import hash_aware_top_b200 as H

    return H


def test_noalloc_rejects_problems_beyond_its_scratch(H):
    """Oversized problems fail on the host with HATA_ERR_WORKSPACE (no launch, no allocation)."""
    d = H.dims_for(64, 64, 8, 128, 256, 1 << 20, "bf16")  # histograms alone would need hundreds of MiB
    fake = ctypes.c_void_p(0x1000)
    assert H.lib.hata_topk_noalloc(ctypes.byref(d), fake, fake, 16, fake, None, None) == H.HATA_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_matches_workspace_topk_twice():
    import torch

    import hash_aware_top_b200 as H

    B, Hkv, G, r, Lmax, k = 3, 2, 4, 128, 13000, 512
    d = H.dims_for(B, G * Hkv, Hkv, 128, r, Lmax, "bf16")
    lens = torch.tensor([13000, 4096, 9001], dtype=torch.int32, device="cuda")
    ws = torch.empty(H.hata_workspace_size(d, k), dtype=torch.uint8, device="cuda")
    H.hata_workspace_init(ws)
    for call, (seed, nd) in enumerate([(31, None), (32, 3)]):  # second call: heavy ties, same scratch
        scores = torch.from_numpy(random_scores((B, Hkv, Lmax), G * r, seed=seed, n_distinct=nd)).cuda()
        want = torch.full((B, Hkv, k), -7, dtype=torch.int32, device="cuda")
        want_n = torch.zeros(B, dtype=torch.int32, device="cuda")
        H.hata_topk(d, scores, lens, k, want, want_n, ws)
        got = torch.full((B, Hkv, k), -9, dtype=torch.int32, device="cuda")
        got_n = torch.zeros(B, dtype=torch.int32, device="cuda")
        H.hata_topk_noalloc(d, scores, lens, k, got, got_n)
        torch.cuda.synchronize()
        assert np.array_equal(got.cpu().numpy(), want.cpu().numpy()), f"call {call}: indices differ"
        assert np.array_equal(got_n.cpu().numpy(), want_n.cpu().numpy()), f"call {call}: counts differ"
