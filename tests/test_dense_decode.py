"""hata_dense_decode: dense flash-decode over every cached token (the dense
attention the "HATA" paper notes time HATA against).  Parity with the oracle's
exact attention over all L_b tokens, through the C ABI, on shapes that span
several 2048-token splits, a ragged last tile and an empty split."""
import numpy as np
import pytest

import oracle
from hata_inputs import Workload, make_inputs

from hata_testlib import TOL, default_scale, dev_float, max_abs

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def H():
    import hash_aware_top_b200 as H

    return H


def test_dense_rejects_unsupported_before_launch(H):
    import ctypes

    fake = ctypes.c_void_p(0x1000)
    d = H.dims_for(1, 4, 1, 128, 128, 4096, "f32")  # fp32 is not supported by the dense kernel
    n = ctypes.c_size_t(0)
    assert H.lib.hata_dense_workspace_size(ctypes.byref(d), ctypes.byref(n)) == H.HATA_OK and n.value > 0
    assert H.lib.hata_dense_decode(ctypes.byref(d), fake, fake, fake, None, 0.0, fake, fake, n.value,
                                   None) == H.HATA_ERR_UNSUPPORTED
    d = H.dims_for(1, 32, 2, 128, 128, 4096, "bf16")  # 16 query heads per KV head
    assert H.lib.hata_dense_decode(ctypes.byref(d), fake, fake, fake, None, 0.0, fake, fake, n.value,
                                   None) == H.HATA_ERR_UNSUPPORTED
    d = H.dims_for(1, 4, 1, 128, 128, 4096, "bf16")
    assert H.lib.hata_dense_decode(ctypes.byref(d), fake, fake, fake, None, 0.0, fake, fake, 16,
                                   None) == H.HATA_ERR_WORKSPACE


@pytest.mark.gpu
@pytest.mark.parametrize("G", [1, 4, 8])
def test_dense_decode_matches_exact_attention(H, G):
    B, Hkv, Lmax = 2, 2, 5000
    Hq = G * Hkv
    wl = Workload("dense", B, Hq, Hkv, 128, Lmax, 128, 64, "bf16", seq_len_range=(1, Lmax))
    inp = make_inputs(wl, seed=40 + G)
    lens = np.array([5000, 1987], dtype=np.int32)  # 3 splits, ragged tiles; the short one leaves a split empty
    d = H.dims_for(B, Hq, Hkv, 128, 128, Lmax, "bf16")
    ws = torch.zeros(H.hata_dense_workspace_size(d), dtype=torch.uint8, device="cuda")
    out = torch.full((B, Hq, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    scale = default_scale(128)
    q, K, V = dev_float(inp["q"], "bf16"), dev_float(inp["K"], "bf16"), dev_float(inp["V"], "bf16")
    for rep in range(2):  # the second call reuses the counters the first one reset
        H.hata_dense_decode(d, q, K, V, torch.from_numpy(lens).cuda(), scale, out, ws)
        got = out.float().cpu().numpy()
        for b in range(B):
            for g in range(Hkv):
                S = np.arange(lens[b])
                want = oracle.sparse_attention(inp["q"][b, g * G:(g + 1) * G], inp["K"][b, g], inp["V"][b, g], S,
                                               scale)
                assert max_abs(got[b, g * G:(g + 1) * G], want) <= TOL["bf16"], (rep, b, g)
    assert H.hata_read_device_status(ws) == 0


@pytest.mark.gpu
def test_dense_equals_hata_when_k_covers_the_cache(H):
    """With k >= L the HATA step selects every token, so it computes the same
    attention as the dense kernel (within bf16 tolerance of each other)."""
    from hata_testlib import dev_codes, new_workspace

    wl = Workload("dense_k", 1, 8, 2, 128, 3000, 128, 3000, "bf16")
    inp = make_inputs(wl, seed=7)
    codes0, _ = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"])
    d = H.dims_for(1, 8, 2, 128, 128, 3000, "bf16")
    q, K, V = dev_float(inp["q"], "bf16"), dev_float(inp["K"], "bf16"), dev_float(inp["V"], "bf16")
    lens = torch.from_numpy(inp["seq_lens"]).cuda()
    out_h = torch.empty((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    H.hata_decode_step(d, q, K, V, torch.from_numpy(inp["W_H"]).cuda(), dev_codes(codes0), lens, 3000, 0.0, out_h,
                       None, None, new_workspace(d, 3000))
    out_d = torch.empty_like(out_h)
    ws = torch.zeros(H.hata_dense_workspace_size(d), dtype=torch.uint8, device="cuda")
    H.hata_dense_decode(d, q, K, V, lens, 0.0, out_d, ws)
    assert max_abs(out_h.float().cpu().numpy(), out_d.float().cpu().numpy()) <= TOL["bf16"]
