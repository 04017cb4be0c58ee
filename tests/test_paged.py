"""The decode step over a paged cache (pools of blocks plus a block table, the
layout of vLLM PagedAttention, which the HashAttention summary lists among its
foundations), against the oracle run on the same data laid out densely; and a
growing cache decoded step by step, one appended token per step."""
import math

import numpy as np
import pytest
import torch

import oracle
from hata_inputs import Workload, make_inputs

from hata_testlib import assert_codes_match, dev_float, max_abs, new_workspace, TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import hash_aware_top_b200 as H

    return H


def block_table_for(B, max_blocks, n_spare, seed):
    """A random, non-contiguous assignment of pool blocks; n_spare blocks stay unused."""
    perm = np.random.default_rng(seed).permutation(B * max_blocks + n_spare).astype(np.int32)
    return perm[: B * max_blocks].reshape(B, max_blocks), B * max_blocks + n_spare


def to_pool(dense, bt, n_blocks, bs, fill):
    """[B][Hkv][Lmax][X] -> [n_blocks][Hkv][bs][X] following the block table; unused slots hold `fill`."""
    B, Hkv, Lmax, X = dense.shape
    pool = np.empty((n_blocks, Hkv, bs, X), dtype=dense.dtype)
    pool[...] = fill
    for b in range(B):
        for i in range(bt.shape[1]):
            lo, hi = i * bs, min(Lmax, (i + 1) * bs)
            if lo < hi:
                pool[bt[b, i], :, : hi - lo] = dense[b, :, lo:hi]
    return pool


def from_pool(pool, bt, Lmax):
    n_blocks, Hkv, bs, X = pool.shape
    B = bt.shape[0]
    dense = np.zeros((B, Hkv, Lmax, X), dtype=pool.dtype)
    for b in range(B):
        for i in range(bt.shape[1]):
            lo, hi = i * bs, min(Lmax, (i + 1) * bs)
            if lo < hi:
                dense[b, :, lo:hi] = pool[bt[b, i], :, : hi - lo]
    return dense


def run_paged(H, wl, q, K_pool, V_pool, W_q, W_k, codes_pool, bt, bs, lens, ws=None):
    d = H.dims_for(wl.batch, wl.n_q_heads, wl.n_kv_heads, 128, wl.hash_bits, wl.max_seq, wl.dtype)
    ws = ws if ws is not None else new_workspace(d, wl.k)
    out = torch.full((wl.batch, wl.n_q_heads, 128), float("nan"), dtype=d.torch_dtype, device="cuda")
    qcode = torch.zeros((wl.batch, wl.n_q_heads, wl.words), dtype=torch.int32, device="cuda")
    idx = torch.full((wl.batch, wl.n_kv_heads, wl.k), -99, dtype=torch.int32, device="cuda")
    H.hata_decode_step_paged(d, dev_float(q, wl.dtype), K_pool, V_pool, torch.from_numpy(W_q).cuda(),
                             torch.from_numpy(W_k).cuda(), codes_pool, torch.from_numpy(bt).cuda(), bs,
                             torch.from_numpy(lens).cuda(), wl.k, 0.0, out, qcode, idx, ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), qcode.cpu().numpy().view(np.uint32), idx.cpu().numpy(), ws


def check_against_oracle(wl, q, K, V, W_q, W_k, codes_before, lens, codes_after, out, qcode, idx):
    """One step against the oracle on the dense view (validity check with the GPU's codes
    where a projection fell inside the sign-exemption band)."""
    ref = oracle.decode_step(q, K, V, W_q, codes_before, lens, wl.k, W_k=W_k)
    G, r = wl.group, wl.hash_bits
    flips = assert_codes_match(qcode, ref["qcode"], ref["y_q"], r)
    for b in range(wl.batch):
        Lb = int(lens[b])
        for g in range(wl.n_kv_heads):
            flips += assert_codes_match(codes_after[b, g, Lb - 1], ref["codes"][b, g, Lb - 1], ref["y_k"][b, g], r)
            assert np.array_equal(codes_after[b, g, : Lb - 1], codes_before[b, g, : Lb - 1])
    for b in range(wl.batch):
        Lb = int(lens[b])
        for g in range(wl.n_kv_heads):
            hs = slice(g * G, (g + 1) * G)
            if flips == 0:
                want_idx, want_out = ref["idx"][b, g], ref["out"][b, hs]
            else:
                D = oracle.gqa_scores(qcode[b, hs], codes_after[b, g, :Lb], r)
                S = oracle.topk_select(D, wl.k)
                want_idx = np.full(wl.k, -1)
                want_idx[: len(S)] = S
                want_out = oracle.sparse_attention(q[b, hs], K[b, g], V[b, g], S, 1 / math.sqrt(128))
            assert np.array_equal(idx[b, g], want_idx), (b, g)
            assert max_abs(out[b, hs], want_out) <= TOL[wl.dtype], (b, g)


PAGED_CASES = [
    (Workload("llama_9k", 1, 32, 8, 128, 9000, 128, 512, "bf16"), 256, False),
    (Workload("ragged_b3", 3, 8, 2, 128, 12000, 128, 1024, "bf16", seq_len_range=(300, 12000)), 128, True),
    (Workload("narrow32", 2, 8, 2, 128, 8192, 32, 256, "bf16", seq_len_range=(5000, 8192)), 64, False),
    (Workload("tiny_f32", 1, 1, 1, 128, 4096, 128, 256, "f32", n_planted=40), 16, True),
]


@pytest.mark.parametrize("case", range(len(PAGED_CASES)))
def test_paged_step_matches_oracle(H, case):
    wl, bs, separate_k = PAGED_CASES[case]
    inp = make_inputs(wl, seed=23)
    W_q = inp["W_H"]
    W_k = (np.random.default_rng(2323).standard_normal(W_q.shape) / math.sqrt(128)).astype(np.float32) \
        if separate_k else W_q
    codes0, _ = oracle.encode_cache(inp["K"], W_k, inp["seq_lens"])
    max_blocks = (wl.max_seq + bs - 1) // bs
    bt, n_blocks = block_table_for(wl.batch, max_blocks, 5, seed=case)
    garbage = np.float32(1e30)  # unused slots: a read of one would wreck the outputs
    K_pool = dev_float(to_pool(inp["K"], bt, n_blocks, bs, garbage), wl.dtype)
    V_pool = dev_float(to_pool(inp["V"], bt, n_blocks, bs, garbage), wl.dtype)
    codes_pool = torch.from_numpy(to_pool(codes0, bt, n_blocks, bs, 0xA5A5A5A5).view(np.int32)).cuda()
    out, qcode, idx, ws = run_paged(H, wl, inp["q"], K_pool, V_pool, W_q, W_k, codes_pool, bt, bs, inp["seq_lens"])
    codes_after = from_pool(codes_pool.cpu().numpy().view(np.uint32), bt, wl.max_seq)
    check_against_oracle(wl, inp["q"], inp["K"], inp["V"], W_q, W_k, codes0, inp["seq_lens"], codes_after, out,
                         qcode, idx)
    assert H.hata_read_device_status(ws) == 0


def test_paged_growing_cache_multi_step(H):
    """Six decode steps over one paged cache: every step appends one token (its K/V
    row already in its slot), the step writes that token's code into its page, and
    the next step scans it.  Each step matches the oracle on the dense view."""
    wl = Workload("grow", 2, 8, 2, 128, 1500, 128, 64, "bf16", seq_len_range=(900, 1300))
    bs = 64
    inp = make_inputs(wl, seed=29)
    L0 = inp["seq_lens"].copy()
    W = inp["W_H"]
    codes = oracle.encode_cache(inp["K"], W, L0, upto_last=False)[0]  # slots [0, L0) cached
    max_blocks = (wl.max_seq + bs - 1) // bs
    bt, n_blocks = block_table_for(wl.batch, max_blocks, 3, seed=7)
    K_pool = dev_float(to_pool(inp["K"], bt, n_blocks, bs, 0.0), wl.dtype)
    V_pool = dev_float(to_pool(inp["V"], bt, n_blocks, bs, 0.0), wl.dtype)
    codes_pool = torch.from_numpy(to_pool(codes, bt, n_blocks, bs, 0).view(np.int32)).cuda()
    rng = np.random.default_rng(31)
    ws = None
    for step in range(6):
        lens = (L0 + step + 1).astype(np.int32)
        q = torch.tensor(rng.standard_normal(inp["q"].shape, dtype=np.float32)).bfloat16().float().numpy()
        out, qcode, idx, ws = run_paged(H, wl, q, K_pool, V_pool, W, W, codes_pool, bt, bs, lens, ws=ws)
        codes_after = from_pool(codes_pool.cpu().numpy().view(np.uint32), bt, wl.max_seq)
        check_against_oracle(wl, q, inp["K"], inp["V"], W, W, codes, lens, codes_after, out, qcode, idx)
        codes = codes_after  # the cache as the GPU left it (codes inside the exemption band included)
    assert H.hata_read_device_status(ws) == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_append_kv_paged(H, dtype):
    """The paged cache update writes each new row to the slot the block table gives for
    position L_b - 1 (compared on the dense view with oracle.append_kv), and nothing else;
    lengths 0 and max_seq + 1 and a block number outside the pool write nothing."""
    B, Hkv, Lmax, bs = 5, 2, 300, 64
    rng = np.random.default_rng(41)
    K0 = rng.standard_normal((B, Hkv, Lmax, 128)).astype(np.float32)
    V0 = rng.standard_normal((B, Hkv, Lmax, 128)).astype(np.float32)
    nk = rng.standard_normal((B, Hkv, 128)).astype(np.float32)
    nv = rng.standard_normal((B, Hkv, 128)).astype(np.float32)
    lens = np.array([1, 300, 0, 301, 130], dtype=np.int32)
    max_blocks = (Lmax + bs - 1) // bs
    bt, n_blocks = block_table_for(B, max_blocks, 2, seed=43)
    bt_dev = bt.copy()
    bt_dev[4, 129 // bs] = n_blocks + 5  # batch 4's page of position 129: outside the pool
    d = H.dims_for(B, 2 * Hkv, Hkv, 128, 128, Lmax, dtype)
    rnd = lambda a: dev_float(a, dtype).float().cpu().numpy()  # noqa: E731  (the device's rounding)
    K0, V0, nk, nv = rnd(K0), rnd(V0), rnd(nk), rnd(nv)
    Kp = dev_float(to_pool(K0, bt, n_blocks, bs, 0.0), dtype)
    Vp = dev_float(to_pool(V0, bt, n_blocks, bs, 0.0), dtype)
    H.hata_append_kv_paged(d, dev_float(nk, dtype), dev_float(nv, dtype), Kp, Vp, torch.from_numpy(bt_dev).cuda(), bs,
                           torch.from_numpy(lens).cuda())
    torch.cuda.synchronize()
    want_lens = lens.copy()
    want_lens[4] = 0  # its block number is outside the pool: nothing written
    K2, V2 = oracle.append_kv(K0, V0, nk, nv, want_lens)
    assert np.array_equal(from_pool(Kp.float().cpu().numpy(), bt, Lmax), K2)
    assert np.array_equal(from_pool(Vp.float().cpu().numpy(), bt, Lmax), V2)
