"""GPU parity: every CUDA entry point against the CPU oracle, element by element,
on seeded inputs small enough for the oracle but spanning several CTA tiles and
a ragged tail.  All calls go through the C ABI (binding -> libhata.so)."""
import math

import numpy as np
import pytest

import oracle
from hata_inputs import Workload, make_inputs, random_codes, random_indices, random_scores

from hata_testlib import (TOL, assert_codes_match, check_step, default_scale, dev_codes, dev_float, host_codes,
                          max_abs, new_workspace, run_step)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def H():
    import hash_aware_top_b200 as H

    return H


def _dims(H, B, Hq, Hkv, r, Lmax, dtype):
    return H.dims_for(B, Hq, Hkv, 128, r, Lmax, dtype)


# ----------------------------------------------------------------------------
# HashEncode
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("r", [32, 64, 128, 256])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_encode_prefill_and_queries(H, r, dtype):
    wl = Workload("enc", 2, 8, 2, 128, 1000, r, 16, dtype, seq_len_range=(700, 1000))
    inp = make_inputs(wl, seed=1)
    d = _dims(H, 2, 8, 2, r, 1000, dtype)
    K = dev_float(inp["K"], dtype)
    W = torch.from_numpy(inp["W_H"]).cuda()
    lens = torch.from_numpy(inp["seq_lens"]).cuda()
    sentinel = np.uint32(0xA5A5A5A5)
    codes = dev_codes(np.full((2, 2, 1000, r // 32), sentinel, dtype=np.uint32))
    # prefill every slot below L_b: n_tok = max_seq ending at seq_lens
    ws = new_workspace(d, 16)
    H.hata_encode_append(d, K, 2, 1000, 1000, lens, W, codes, 1000, ws)
    assert H.hata_read_device_status(ws) == 0
    got = host_codes(codes)
    want, ys = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"], upto_last=False)
    for b in range(2):
        Lb = int(inp["seq_lens"][b])
        for g in range(2):
            assert_codes_match(got[b, g, :Lb], want[b, g, :Lb], ys[(b, g)], r)
            assert np.all(got[b, g, Lb:] == sentinel), "slots beyond L_b must not be written"
    # queries: x_len = codes_len = 1, heads grouped on W_H[h // G]
    q = dev_float(inp["q"], dtype)
    qc = dev_codes(np.zeros((2, 8, r // 32), dtype=np.uint32))
    H.hata_encode_append(d, q, 8, 1, 1, None, W, qc, 1, ws)
    gq = host_codes(qc)
    for b in range(2):
        for h in range(8):
            c, y = oracle.encode(inp["q"][b, h], inp["W_H"][h // 4])
            assert_codes_match(gq[b, h], c, y, r)


@pytest.mark.parametrize("r", [32, 64, 128])
def test_encode_prefill_many_tiles_per_cta(H, r):
    """A prefill long enough that every CTA of the tensor-core encode runs many
    128-key tiles (its shared-memory stages and both accumulators wrap around
    several times), with a ragged end."""
    B, Hkv, L = 1, 8, 40000
    wl = Workload("enc_long", B, 8, Hkv, 128, L, r, 16, "bf16", seq_len_range=(L - 77, L - 77))
    inp = make_inputs(wl, seed=3, plant=False)
    d = _dims(H, B, 8, Hkv, r, L, "bf16")
    codes = dev_codes(np.zeros((B, Hkv, L, r // 32), dtype=np.uint32))
    ws = new_workspace(d, 16)
    H.hata_encode_append(d, dev_float(inp["K"], "bf16"), Hkv, L, L, torch.from_numpy(inp["seq_lens"]).cuda(),
                         torch.from_numpy(inp["W_H"]).cuda(), codes, L, ws)
    assert H.hata_read_device_status(ws) == 0
    got = host_codes(codes)
    want, ys = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"], upto_last=False)
    Lb = int(inp["seq_lens"][0])
    for g in range(Hkv):
        assert_codes_match(got[0, g, :Lb], want[0, g, :Lb], ys[(0, g)], r)
        assert np.all(got[0, g, Lb:] == 0)


def test_encode_prefill_grouped_heads_window(H):
    """The prefill form on query-like input: x_heads = Hq grouped on W_H[h // G],
    a window of n_tok slots ending at seq_end, codes_len shorter than x_len."""
    B, Hq, Hkv, xl, cl, r = 2, 8, 2, 700, 650, 128
    rng = np.random.default_rng(5)
    x = torch.tensor(rng.standard_normal((B, Hq, xl, 128), dtype=np.float32)).bfloat16()
    W = (rng.standard_normal((Hkv, 128, r)) / math.sqrt(128)).astype(np.float32)
    end = np.array([600, 690], dtype=np.int32)
    n_tok = 333
    d = _dims(H, B, Hq, Hkv, r, cl, "bf16")
    sentinel = np.uint32(0x5A5A5A5A)
    codes = dev_codes(np.full((B, Hq, cl, r // 32), sentinel, dtype=np.uint32))
    ws = new_workspace(d, 16)
    H.hata_encode_append(d, x.cuda(), Hq, xl, n_tok, torch.from_numpy(end).cuda(), torch.from_numpy(W).cuda(),
                         codes, cl, ws)
    assert H.hata_read_device_status(ws) == 0
    got = host_codes(codes)
    xf = x.float().numpy()
    for b in range(B):
        lo, hi = max(int(end[b]) - n_tok, 0), min(int(end[b]), cl)
        for h in range(Hq):
            c, y = oracle.encode(xf[b, h, lo:hi], W[h // (Hq // Hkv)])
            assert_codes_match(got[b, h, lo:hi], c, y, r)
            assert np.all(got[b, h, :lo] == sentinel) and np.all(got[b, h, hi:] == sentinel)


def test_encode_append_single_slot(H):
    """n_tok = 1 at seq_end = seq_lens writes exactly slot L_b - 1."""
    wl = Workload("app", 3, 4, 4, 128, 300, 128, 8, "bf16", seq_len_range=(1, 300))
    inp = make_inputs(wl, seed=2)
    d = _dims(H, 3, 4, 4, 128, 300, "bf16")
    codes0 = random_codes((3, 4, 300), 128, seed=5)
    codes = dev_codes(codes0)
    ws = new_workspace(d, 16)
    H.hata_encode_append(d, dev_float(inp["K"], "bf16"), 4, 300, 1, torch.from_numpy(inp["seq_lens"]).cuda(),
                         torch.from_numpy(inp["W_H"]).cuda(), codes, 300, ws)
    assert H.hata_read_device_status(ws) == 0
    got = host_codes(codes)
    for b in range(3):
        Lb = int(inp["seq_lens"][b])
        for g in range(4):
            c, y = oracle.encode(inp["K"][b, g, Lb - 1], inp["W_H"][g])
            assert_codes_match(got[b, g, Lb - 1], c, y, 128)
            mask = np.ones(300, bool)
            mask[Lb - 1] = False
            assert np.array_equal(got[b, g][mask], codes0[b, g][mask])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_append_kv(H, dtype):
    """The cache update writes the new rows at slot L_b - 1, bit for bit, and nothing else;
    lengths 0 and max_seq + 1 write nothing, lengths 1 and max_seq write the first and last slots."""
    B, Hkv, Lmax = 6, 3, 257
    rng = np.random.default_rng(17)
    K0 = rng.standard_normal((B, Hkv, Lmax, 128)).astype(np.float32)
    V0 = rng.standard_normal((B, Hkv, Lmax, 128)).astype(np.float32)
    nk = rng.standard_normal((B, Hkv, 128)).astype(np.float32)
    nv = rng.standard_normal((B, Hkv, 128)).astype(np.float32)
    lens = np.array([1, Lmax, 0, Lmax + 1, 100, 2], dtype=np.int32)
    d = _dims(H, B, 2 * Hkv, Hkv, 128, Lmax, dtype)
    K, V = dev_float(K0, dtype), dev_float(V0, dtype)
    nkd, nvd = dev_float(nk, dtype), dev_float(nv, dtype)
    H.hata_append_kv(d, nkd, nvd, K, V, torch.from_numpy(lens).cuda())
    # the expected caches, built by the oracle from the same (device-rounded) values
    K2, V2 = oracle.append_kv(dev_float(K0, dtype).float().cpu().numpy(), dev_float(V0, dtype).float().cpu().numpy(),
                              nkd.float().cpu().numpy(), nvd.float().cpu().numpy(), lens)
    assert np.array_equal(K.float().cpu().numpy(), K2)
    assert np.array_equal(V.float().cpu().numpy(), V2)


# ----------------------------------------------------------------------------
# Hamming + GQA sum
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("r", [32, 64, 128, 256])
@pytest.mark.parametrize("G", [1, 2, 3, 4, 8])
def test_hamming_scores(H, r, G):
    B, Hkv, Lmax = 2, 2, 9000
    d = _dims(H, B, G * Hkv, Hkv, r, Lmax, "bf16")
    qcode = random_codes((B, G * Hkv), r, seed=10 + G)
    codes = random_codes((B, Hkv, Lmax), r, seed=20 + r)
    lens = np.array([9000, 4097], dtype=np.int32)
    sc = torch.full((B, Hkv, Lmax), -7, dtype=torch.int32, device="cuda")
    H.hata_hamming_scores(d, dev_codes(qcode), dev_codes(codes), torch.from_numpy(lens).cuda(), sc)
    got = sc.cpu().numpy()
    for b in range(B):
        for g in range(Hkv):
            want = oracle.gqa_scores(qcode[b, g * G:(g + 1) * G], codes[b, g, :lens[b]], r)
            assert np.array_equal(got[b, g, :lens[b]], want)
            assert np.all(got[b, g, lens[b]:] == -7)


def test_hamming_extremes(H):
    """Identical and complementary codes: scores 0 and G * r."""
    d = _dims(H, 1, 4, 1, 128, 64, "bf16")
    q = random_codes((1, 1), 128, seed=3)
    qcode = np.repeat(q, 4, axis=1)
    codes = np.zeros((1, 1, 64, 4), dtype=np.uint32)
    codes[0, 0, ::2] = q[0, 0]
    codes[0, 0, 1::2] = ~q[0, 0]
    sc = torch.zeros((1, 1, 64), dtype=torch.int32, device="cuda")
    H.hata_hamming_scores(d, dev_codes(qcode), dev_codes(codes), torch.tensor([64], dtype=torch.int32).cuda(), sc)
    got = sc.cpu().numpy()[0, 0]
    assert np.all(got[::2] == 0) and np.all(got[1::2] == 4 * 128)


# ----------------------------------------------------------------------------
# Top-k
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("k", [1, 100, 512, 4096, 5000, 20000])
@pytest.mark.parametrize("n_distinct", [None, 3])
def test_topk(H, k, n_distinct):
    B, Hkv, G, r, Lmax = 3, 2, 4, 128, 13000
    d = _dims(H, B, G * Hkv, Hkv, r, Lmax, "bf16")
    scores = random_scores((B, Hkv, Lmax), G * r, seed=k, n_distinct=n_distinct)
    lens = np.array([13000, 4096, 9001], dtype=np.int32)
    ws = new_workspace(d, k)
    idx = torch.full((B, Hkv, k), -99, dtype=torch.int32, device="cuda")
    n_sel = torch.zeros(B, dtype=torch.int32, device="cuda")
    H.hata_topk(d, torch.from_numpy(scores).cuda(), torch.from_numpy(lens).cuda(), k, idx, n_sel, ws)
    got = idx.cpu().numpy()
    for b in range(B):
        for g in range(Hkv):
            S = oracle.topk_select(scores[b, g, :lens[b]], k)
            want = np.full(k, -1)
            want[:len(S)] = S
            assert np.array_equal(got[b, g], want), (b, g)
    assert n_sel.cpu().numpy().tolist() == [min(k, int(x)) for x in lens]
    assert H.hata_read_device_status(ws) == 0


def test_topk_all_equal_and_tiny_lengths(H):
    B, Hkv, Lmax, k = 4, 1, 5000, 7
    d = _dims(H, B, 4, Hkv, 128, Lmax, "bf16")
    scores = np.full((B, Hkv, Lmax), 77, dtype=np.int32)
    lens = np.array([5000, 1, 0, 7], dtype=np.int32)
    ws = new_workspace(d, k)
    idx = torch.full((B, Hkv, k), -99, dtype=torch.int32, device="cuda")
    n_sel = torch.zeros(B, dtype=torch.int32, device="cuda")
    H.hata_topk(d, torch.from_numpy(scores).cuda(), torch.from_numpy(lens).cuda(), k, idx, n_sel, ws)
    got = idx.cpu().numpy()[:, 0]
    assert got[0].tolist() == list(range(7))
    assert got[1].tolist() == [0] + [-1] * 6
    assert got[2].tolist() == [-1] * 7
    assert got[3].tolist() == list(range(7))
    assert n_sel.cpu().numpy().tolist() == [7, 1, 0, 7]


def test_topk_repeated_calls_reuse_workspace(H):
    """Counters are left at zero: the same workspace serves back-to-back calls."""
    B, Hkv, Lmax, k = 1, 8, 20000, 512
    d = _dims(H, B, 32, Hkv, 128, Lmax, "bf16")
    ws = new_workspace(d, k)
    lens = torch.tensor([20000], dtype=torch.int32).cuda()
    for seed in range(3):
        scores = random_scores((B, Hkv, Lmax), 512, seed=seed)
        idx = torch.empty((B, Hkv, k), dtype=torch.int32, device="cuda")
        H.hata_topk(d, torch.from_numpy(scores).cuda(), lens, k, idx, None, ws)
        got = idx.cpu().numpy()
        for g in range(Hkv):
            assert np.array_equal(got[0, g], oracle.topk_select(scores[0, g], k))


# ----------------------------------------------------------------------------
# Sparse decode
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("k", [1, 33, 512, 1000])
def test_sparse_decode(H, dtype, k):
    B, Hq, Hkv, Lmax = 2, 8, 2, 3000
    wl = Workload("sd", B, Hq, Hkv, 128, Lmax, 128, k, dtype, seq_len_range=(1, 3000))
    inp = make_inputs(wl, seed=k)
    lens = np.array([3000, 700], dtype=np.int32)
    idx = random_indices(B * Hkv, np.repeat(lens, Hkv), k, seed=k).reshape(B, Hkv, k)
    d = _dims(H, B, Hq, Hkv, 128, Lmax, dtype)
    ws = new_workspace(d, k)
    out = torch.full((B, Hq, 128), float("nan"), dtype=d.torch_dtype, device="cuda")
    scale = default_scale(128)
    H.hata_sparse_decode(d, dev_float(inp["q"], dtype), dev_float(inp["K"], dtype), dev_float(inp["V"], dtype),
                         torch.from_numpy(idx).cuda(), k, scale, out, ws)
    got = out.float().cpu().numpy()
    G = Hq // Hkv
    for b in range(B):
        for g in range(Hkv):
            S = idx[b, g][idx[b, g] >= 0]
            want = oracle.sparse_attention(inp["q"][b, g * G:(g + 1) * G], inp["K"][b, g], inp["V"][b, g], S, scale)
            assert max_abs(got[b, g * G:(g + 1) * G], want) <= TOL[dtype]
    assert H.hata_read_device_status(ws) == 0


def test_sparse_decode_empty_selection_and_bad_index(H):
    d = _dims(H, 1, 4, 1, 128, 64, "f32")
    k = 40
    q = torch.randn(1, 4, 128, device="cuda")
    K = torch.randn(1, 1, 64, 128, device="cuda")
    V = torch.randn(1, 1, 64, 128, device="cuda")
    ws = new_workspace(d, k)
    out = torch.full((1, 4, 128), float("nan"), device="cuda")
    idx = torch.full((1, 1, k), -1, dtype=torch.int32, device="cuda")
    H.hata_sparse_decode(d, q, K, V, idx, k, 0.0, out, ws)
    assert torch.all(out == 0)
    idx[0, 0, 0] = 5
    idx[0, 0, 1] = 64  # outside the cache: skipped and flagged
    H.hata_sparse_decode(d, q, K, V, idx, k, 0.0, out, ws)
    assert torch.allclose(out[0], V[0, 0, 5].expand(4, 128))
    assert H.hata_read_device_status(ws) == H.HATA_ERR_INVALID_ARG
    assert H.hata_read_device_status(ws) == 0


# ----------------------------------------------------------------------------
# Whole decode step
# ----------------------------------------------------------------------------

STEP_CASES = {
    "tiny_f32_4k": Workload("tiny_f32_4k", 1, 1, 1, 128, 4096, 128, 256, "f32", n_planted=40),
    "llama_shape_9k": Workload("llama_shape_9k", 1, 32, 8, 128, 9000, 128, 512, "bf16"),
    "ragged_b3": Workload("ragged_b3", 3, 8, 2, 128, 12000, 128, 1024, "bf16", seq_len_range=(300, 12000)),
    "narrow32": Workload("narrow32", 2, 8, 2, 128, 8192, 32, 256, "bf16", seq_len_range=(5000, 8192)),
    "g3_chain": Workload("g3_chain", 2, 6, 2, 128, 3000, 128, 100, "bf16", seq_len_range=(1500, 3000)),
    "short_lens": Workload("short_lens", 6, 8, 2, 128, 64, 128, 16, "bf16", seq_len_range=(1, 64), n_planted=2),
    "budget_gt_slice": Workload("budget_gt_slice", 1, 8, 2, 128, 3000, 128, 2048, "f32"),
    "r32_g8_f32": Workload("r32_g8_f32", 2, 16, 2, 128, 6000, 32, 300, "f32", seq_len_range=(3001, 6000)),
    # many units -> small clusters with more than 8192 tokens per CTA (multi-pass selection)
    "many_units_fallback": Workload("many_units_fallback", 16, 8, 2, 128, 40000, 128, 600, "bf16",
                                    seq_len_range=(20000, 40000)),
    "many_units_covered": Workload("many_units_covered", 16, 8, 2, 128, 40000, 128, 40, "bf16",
                                   seq_len_range=(20000, 40000)),
    "narrow_many_units": Workload("narrow_many_units", 8, 16, 4, 128, 30000, 32, 900, "bf16",
                                  seq_len_range=(15001, 30000)),
    "r64_g2": Workload("r64_g2", 2, 4, 2, 128, 5000, 64, 300, "f32"),
    "r256_g8": Workload("r256_g8", 1, 8, 1, 128, 5000, 256, 128, "bf16"),
    # longer caches with few units, a budget far above a CTA's share, narrow fp32 codes
    "llama_shape_20k": Workload("llama_shape_20k", 1, 32, 8, 128, 20000, 128, 512, "bf16"),
    "ragged_24k": Workload("ragged_24k", 2, 16, 4, 128, 24000, 128, 700, "bf16", seq_len_range=(9000, 24000)),
    "big_k_20k": Workload("big_k_20k", 1, 8, 2, 128, 20000, 128, 4096, "bf16"),
    "r32_f32_17k": Workload("r32_f32_17k", 1, 8, 2, 128, 17000, 32, 500, "f32", seq_len_range=(16500, 17000)),
}


FORMS = {"auto": 0, "all_sm": 4}  # the planner's choice, and the all-SM form forced (HATA_FLAG_ALL_SM_SCAN)


@pytest.mark.parametrize("form", list(FORMS))
@pytest.mark.parametrize("name", list(STEP_CASES))
def test_decode_step(H, name, form):
    wl = STEP_CASES[name]
    inp = make_inputs(wl, seed=7)
    codes0, _ = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"])
    got = run_step(H, wl, inp, codes0, flags=FORMS[form])
    check_step(wl, inp, codes0, got)
    assert H.hata_read_device_status(got["ws"]) == 0


@pytest.mark.parametrize("form", list(FORMS))
def test_decode_step_equals_granular_chain(H, form):
    """Both fused forms and the chain of granular calls agree bit for bit in codes and indices."""
    wl = STEP_CASES["ragged_b3"]
    inp = make_inputs(wl, seed=9)
    codes0, _ = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"])
    fused = run_step(H, wl, inp, codes0, flags=FORMS[form])
    d = H.dims_for(wl.batch, wl.n_q_heads, wl.n_kv_heads, 128, wl.hash_bits, wl.max_seq, wl.dtype)
    ws = new_workspace(d, wl.k)
    q, K, V = (dev_float(inp[n], wl.dtype) for n in ("q", "K", "V"))
    W = torch.from_numpy(inp["W_H"]).cuda()
    lens = torch.from_numpy(inp["seq_lens"]).cuda()
    codes = dev_codes(codes0)
    qc = torch.zeros((wl.batch, wl.n_q_heads, wl.words), dtype=torch.int32, device="cuda")
    H.hata_encode_append(d, q, wl.n_q_heads, 1, 1, None, W, qc, 1, ws)
    H.hata_encode_append(d, K, wl.n_kv_heads, wl.max_seq, 1, lens, W, codes, wl.max_seq, ws)
    sc = torch.empty((wl.batch, wl.n_kv_heads, wl.max_seq), dtype=torch.int32, device="cuda")
    H.hata_hamming_scores(d, qc, codes, lens, sc)
    idx = torch.empty((wl.batch, wl.n_kv_heads, wl.k), dtype=torch.int32, device="cuda")
    H.hata_topk(d, sc, lens, wl.k, idx, None, ws)
    out = torch.empty((wl.batch, wl.n_q_heads, 128), dtype=d.torch_dtype, device="cuda")
    H.hata_sparse_decode(d, q, K, V, idx, wl.k, 0.0, out, ws)
    assert np.array_equal(host_codes(qc), fused["qcode"])
    assert np.array_equal(host_codes(codes), fused["codes"])
    assert np.array_equal(idx.cpu().numpy(), fused["idx"])
    assert max_abs(out.float().cpu().numpy(), fused["out"]) <= TOL[wl.dtype]


def test_decode_step_without_debug_outputs_and_repeat(H):
    wl = STEP_CASES["llama_shape_9k"]
    inp = make_inputs(wl, seed=11)
    codes0, _ = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"])
    a = run_step(H, wl, inp, codes0, with_debug=True)
    b = run_step(H, wl, inp, codes0, ws=a["ws"], with_debug=False)
    assert np.array_equal(a["out"], b["out"])
    assert np.array_equal(a["codes"], b["codes"])


def run_step_qk(H, wl, inp, W_k, codes0, ws=None):
    d = H.dims_for(wl.batch, wl.n_q_heads, wl.n_kv_heads, 128, wl.hash_bits, wl.max_seq, wl.dtype)
    ws = ws if ws is not None else new_workspace(d, wl.k)
    codes = dev_codes(codes0, wl.hash_bits)
    out = torch.full((wl.batch, wl.n_q_heads, 128), float("nan"), dtype=d.torch_dtype, device="cuda")
    qcode = torch.zeros(d.code_shape(wl.batch, wl.n_q_heads), dtype=torch.int16 if wl.hash_bits == 16 else torch.int32,
                        device="cuda")
    idx = torch.full((wl.batch, wl.n_kv_heads, wl.k), -99, dtype=torch.int32, device="cuda")
    H.hata_decode_step_qk(d, dev_float(inp["q"], wl.dtype), dev_float(inp["K"], wl.dtype),
                          dev_float(inp["V"], wl.dtype), torch.from_numpy(inp["W_H"]).cuda(),
                          torch.from_numpy(W_k).cuda(), codes, torch.from_numpy(inp["seq_lens"]).cuda(), wl.k, 0.0,
                          out, qcode, idx, ws)
    torch.cuda.synchronize()
    return {"codes": host_codes(codes), "out": out.float().cpu().numpy(), "qcode": host_codes(qcode),
            "idx": idx.cpu().numpy(), "ws": ws}


@pytest.mark.parametrize("name", ["llama_shape_9k", "narrow32", "tiny_f32_4k", "ragged_b3", "g3_chain"])
def test_decode_step_separate_key_encoder(H, name):
    """HashAttention form: queries encoded with W_q (= the workload's W_H), keys
    with an independent W_k; the cache holds W_k codes.  Fused shapes and the
    granular chain (g3_chain) against the oracle."""
    wl = STEP_CASES[name]
    inp = make_inputs(wl, seed=17)
    W_k = (np.random.default_rng(1717).standard_normal(inp["W_H"].shape) / math.sqrt(128)).astype(np.float32)
    codes0, _ = oracle.encode_cache(inp["K"], W_k, inp["seq_lens"])
    got = run_step_qk(H, wl, inp, W_k, codes0)
    check_step(wl, inp, codes0, got, W_k=W_k)
    assert H.hata_read_device_status(got["ws"]) == 0


def test_decode_step_qk_with_one_encoder_equals_decode_step(H):
    wl = STEP_CASES["llama_shape_9k"]
    inp = make_inputs(wl, seed=19)
    codes0, _ = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"])
    a = run_step(H, wl, inp, codes0)
    b = run_step_qk(H, wl, inp, inp["W_H"].copy(), codes0)  # a separate buffer holding the same matrix
    for k_ in ("codes", "qcode", "idx", "out"):
        assert np.array_equal(a[k_], b[k_]), k_


def test_decode_step_flags_length_beyond_cache(H):
    wl = Workload("bad", 1, 4, 1, 128, 256, 128, 16, "bf16")
    inp = make_inputs(wl, seed=1)
    inp["seq_lens"] = np.array([300], dtype=np.int32)  # > max_seq: clamped and flagged
    codes0 = random_codes((1, 1, 256), 128, seed=2)
    got = run_step(H, wl, inp, codes0)
    assert H.hata_read_device_status(got["ws"]) == H.HATA_ERR_INVALID_ARG


def test_kernel_count_reports_the_form(H):
    # the cluster form (one launch), the all-SM form (encode, scan and tail kernels),
    # and the chain of six granular launches (G = 3)
    assert H.hata_decode_step_kernel_count(H.dims_for(1, 32, 8, 128, 128, 131072, "bf16"), 512) == 1
    assert H.hata_decode_step_kernel_count(H.dims_for(16, 32, 8, 128, 128, 65536, "bf16"), 1024) == 3
    assert H.hata_decode_step_kernel_count(H.dims_for(1, 32, 8, 128, 128, 131072, "bf16", 4), 512) == 3
    # 32 units: the all-SM form once the selection is large (k = 2048), the cluster form for k = 512
    assert H.hata_decode_step_kernel_count(H.dims_for(4, 32, 8, 128, 32, 65536, "bf16"), 2048) == 3
    assert H.hata_decode_step_kernel_count(H.dims_for(4, 32, 8, 128, 32, 65536, "bf16"), 512) == 1
    assert H.hata_decode_step_kernel_count(H.dims_for(1, 6, 2, 128, 128, 3000, "bf16"), 100) == 6


def _custom_step(H, wl, seed, codes0):
    inp = make_inputs(wl, seed=seed, plant=False)
    for flags in FORMS.values():
        got = run_step(H, wl, inp, codes0, flags=flags)
        check_step(wl, inp, codes0, got)
        assert H.hata_read_device_status(got["ws"]) == 0


def test_decode_step_heavy_ties(H):
    """Every cached code equal: all but the new token tie.  The earliest chunks' candidate
    lists cannot hold their tie quota, so the tail kernel rescores them from the cache."""
    wl = Workload("ties", 2, 8, 2, 128, 20000, 128, 600, "bf16", seq_len_range=(15000, 20000))
    codes0 = np.repeat(random_codes((1, 1, 1), 128, seed=3), 2 * 2 * 20000, axis=0).reshape(2, 2, 20000, 4)
    _custom_step(H, wl, 21, codes0)


def test_decode_step_selection_in_one_chunk(H):
    """The k nearest codes all sit in the first 2,000 slots (a copy of the group's first
    query code with a few random bits flipped), so one chunk holds the whole selection and
    its list stops short of the threshold."""
    wl = Workload("clustered", 1, 16, 4, 128, 60000, 128, 700, "bf16")
    inp = make_inputs(wl, seed=23, plant=False)
    qcode = oracle.decode_step(inp["q"], inp["K"], inp["V"], inp["W_H"], np.zeros((1, 4, 60000, 4), np.uint32),
                               inp["seq_lens"], 1)["qcode"]
    codes0 = random_codes((1, 4, 60000), 128, seed=5)
    rng = np.random.default_rng(29)
    for g in range(4):
        near = np.repeat(qcode[0, 4 * g][None, :], 2000, axis=0)
        flips = np.zeros((2000, 4), np.uint32)
        for t in range(2000):  # 1-20 random bit flips per slot: many distinct low scores
            for bit in rng.choice(128, size=int(rng.integers(1, 21)), replace=False):
                flips[t, bit // 32] |= np.uint32(1) << np.uint32(bit % 32)
        codes0[0, g, :2000] = near ^ flips
    _custom_step(H, wl, 23, codes0)
