"""16-bit signatures: the narrowest width of the signature-width ablation in
"HashAttention: Semantic Sparsity for Faster Inference" (16 -> 32 -> 64 bits),
used at sparsity k = L/16 and k = L/32.  A 16-bit code is stored as one uint16
per token (two tokens per 32-bit word, the earlier token in the low half), bit j
of the code at bit j of that value.  The encode (prefill and decode forms), the
Hamming scan with the GQA sum, and the decode step (HATA's single encoder and
the separate query / key encoders) are compared with the oracle through the C ABI.
"""
import math

import numpy as np
import pytest

import oracle
from hata_inputs import Workload, make_inputs, random_codes

from hata_testlib import (assert_codes_match, check_step, dev_codes, dev_float, host_codes, new_workspace,
                          run_step)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def H():
    import hash_aware_top_b200 as H

    return H


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_encode_sixteen_bit_prefill_and_queries(H, dtype):
    wl = Workload("enc16", 2, 8, 2, 128, 1000, 16, 16, dtype, seq_len_range=(700, 1000))
    inp = make_inputs(wl, seed=41)
    d = H.dims_for(2, 8, 2, 128, 16, 1000, dtype)
    ws = new_workspace(d, 16)
    sentinel = np.uint32(0xA5A5)
    codes = dev_codes(np.full((2, 2, 1000, 1), sentinel, dtype=np.uint32), 16)
    H.hata_encode_append(d, dev_float(inp["K"], dtype), 2, 1000, 1000, torch.from_numpy(inp["seq_lens"]).cuda(),
                         torch.from_numpy(inp["W_H"]).cuda(), codes, 1000, ws)
    assert H.hata_read_device_status(ws) == 0
    got = host_codes(codes)
    want, ys = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"], upto_last=False)
    for b in range(2):
        Lb = int(inp["seq_lens"][b])
        for g in range(2):
            assert_codes_match(got[b, g, :Lb], want[b, g, :Lb], ys[(b, g)], 16)
            assert np.all(got[b, g, Lb:] == sentinel), "slots beyond L_b must not be written"
    qc = dev_codes(np.zeros((2, 8, 1), dtype=np.uint32), 16)
    H.hata_encode_append(d, dev_float(inp["q"], dtype), 8, 1, 1, None, torch.from_numpy(inp["W_H"]).cuda(), qc, 1, ws)
    gq = host_codes(qc)
    for b in range(2):
        for h in range(8):
            c, y = oracle.encode(inp["q"][b, h], inp["W_H"][h // 4])
            assert_codes_match(gq[b, h], c, y, 16)


@pytest.mark.parametrize("G", [1, 4, 8])
def test_hamming_sixteen_bit(H, G):
    B, Hkv, Lmax = 2, 2, 5000
    d = H.dims_for(B, G * Hkv, Hkv, 128, 16, Lmax, "bf16")
    qcode = random_codes((B, G * Hkv), 16, seed=43 + G)
    codes = random_codes((B, Hkv, Lmax), 16, seed=47)
    lens = np.array([5000, 1999], dtype=np.int32)
    sc = torch.full((B, Hkv, Lmax), -7, dtype=torch.int32, device="cuda")
    H.hata_hamming_scores(d, dev_codes(qcode, 16), dev_codes(codes, 16), torch.from_numpy(lens).cuda(), sc)
    got = sc.cpu().numpy()
    for b in range(B):
        for g in range(Hkv):
            want = oracle.gqa_scores(qcode[b, g * G:(g + 1) * G], codes[b, g, :lens[b]], 16)
            assert np.array_equal(got[b, g, :lens[b]], want)
            assert np.all(got[b, g, lens[b]:] == -7)


# sparsity 16x and 32x, as in the ablation: k = L / 16 and k = L / 32
SIXTEEN = {
    "L16_llama_shape": Workload("s16a", 1, 32, 8, 128, 16384, 16, 16384 // 16, "bf16"),
    "L32_ragged": Workload("s16b", 3, 8, 2, 128, 12000, 16, 12000 // 32, "bf16", seq_len_range=(4000, 12000)),
    "L16_f32": Workload("s16c", 2, 4, 4, 128, 4096, 16, 4096 // 16, "f32"),
}


@pytest.mark.parametrize("name", list(SIXTEEN))
def test_decode_step_sixteen_bit(H, name):
    wl = SIXTEEN[name]
    inp = make_inputs(wl, seed=51)
    codes0, _ = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"])
    got = run_step(H, wl, inp, codes0)
    check_step(wl, inp, codes0, got)
    assert H.hata_read_device_status(got["ws"]) == 0


@pytest.mark.parametrize("name", ["L16_llama_shape", "L32_ragged"])
def test_decode_step_qk_sixteen_bit(H, name):
    """The HashAttention form at 16 bits: queries encoded with W_q, keys with W_k."""
    wl = SIXTEEN[name]
    inp = make_inputs(wl, seed=53)
    W_k = (np.random.default_rng(5353).standard_normal(inp["W_H"].shape) / math.sqrt(128)).astype(np.float32)
    codes0, _ = oracle.encode_cache(inp["K"], W_k, inp["seq_lens"])
    d = H.dims_for(wl.batch, wl.n_q_heads, wl.n_kv_heads, 128, 16, wl.max_seq, wl.dtype)
    ws = new_workspace(d, wl.k)
    codes = dev_codes(codes0, 16)
    out = torch.full((wl.batch, wl.n_q_heads, 128), float("nan"), dtype=d.torch_dtype, device="cuda")
    qcode = torch.zeros(d.code_shape(wl.batch, wl.n_q_heads), dtype=torch.int16, device="cuda")
    idx = torch.full((wl.batch, wl.n_kv_heads, wl.k), -99, dtype=torch.int32, device="cuda")
    H.hata_decode_step_qk(d, dev_float(inp["q"], wl.dtype), dev_float(inp["K"], wl.dtype),
                          dev_float(inp["V"], wl.dtype), torch.from_numpy(inp["W_H"]).cuda(),
                          torch.from_numpy(W_k).cuda(), codes, torch.from_numpy(inp["seq_lens"]).cuda(), wl.k, 0.0,
                          out, qcode, idx, ws)
    torch.cuda.synchronize()
    got = {"codes": host_codes(codes), "out": out.float().cpu().numpy(), "qcode": host_codes(qcode),
           "idx": idx.cpu().numpy()}
    check_step(wl, inp, codes0, got, W_k=W_k)
    assert H.hata_read_device_status(ws) == 0
