"""Causal prefill attention with the key encode fused in (hata_prefill_attention),
against the oracle: every output row is the oracle's causal attention row
(oracle.prefill_attention_row) within the bf16 tolerance, and every key's code is
the oracle's encoding (oracle.encode_cache over all L_b keys) outside the fp32
rounding band.  Source: HATA paper notes, 整体框架 (prefill: full attention over
the prompt while every key is hashed and cached)."""
import math

import numpy as np
import pytest

import oracle
from hata_inputs import WORKLOADS, Workload, make_inputs, prompt_queries

from hata_testlib import assert_codes_match, dev_codes, dev_float, host_codes

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SENTINEL = 7.0  # out rows t >= L_b keep it
CODE_SENTINEL = 0xA5A5A5A5


@pytest.fixture(scope="module")
def H():
    import hash_aware_top_b200 as H

    return H


def _prompt(wl, seed, q_scale=1.0):
    return np.stack([np.stack([prompt_queries(wl, seed, b, h, q_scale) for h in range(wl.n_q_heads)])
                     for b in range(wl.batch)])


def run_prefill(H, wl, inp, Q, with_codes=True, seq_lens=None, flags=0, nan_tail=False):
    lens = inp["seq_lens"] if seq_lens is None else np.asarray(seq_lens, dtype=np.int32)
    d = H.dims_for(wl.batch, wl.n_q_heads, wl.n_kv_heads, 128, wl.hash_bits, wl.max_seq, "bf16", flags)
    K, V = dev_float(inp["K"], "bf16"), dev_float(inp["V"], "bf16")
    if nan_tail:  # slots at or beyond L_b hold NaN: they must not reach any output
        for b in range(wl.batch):
            K[b, :, int(lens[b]):] = float("nan")
            V[b, :, int(lens[b]):] = float("nan")
    out = torch.full((wl.batch, wl.n_q_heads, wl.max_seq, 128), SENTINEL, dtype=torch.bfloat16, device="cuda")
    codes = None
    if with_codes:
        codes = dev_codes(np.full((wl.batch, wl.n_kv_heads, wl.max_seq, wl.words), CODE_SENTINEL, dtype=np.uint32),
                          wl.hash_bits)
    ws = torch.zeros(H.hata_prefill_workspace_size(d), dtype=torch.uint8, device="cuda")
    H.hata_prefill_attention(d, dev_float(Q, "bf16"), K, V, torch.from_numpy(inp["W_H"]).cuda(), codes,
                             torch.from_numpy(lens).cuda(), 0.0, out, ws)
    torch.cuda.synchronize()
    return {"out": out.float().cpu().numpy(), "codes": host_codes(codes) if with_codes else None,
            "status": H.hata_read_device_status(ws), "lens": lens}


def check_rows(wl, inp, Q, got, rows=None):
    """rows: iterable of (b, h, t); default every valid row.  Tolerance: 1e-2 of the row's
    largest |value| plus 2e-3 (bf16 probabilities and output)."""
    scale = 1.0 / math.sqrt(128)
    lens = got["lens"]
    G = wl.group
    if rows is None:
        rows = [(b, h, t) for b in range(wl.batch) for h in range(wl.n_q_heads) for t in range(int(lens[b]))]
    worst = 0.0
    for b, h, t in rows:
        want = oracle.prefill_attention_row(Q[b, h, t], inp["K"][b, h // G], inp["V"][b, h // G], t, scale)
        err = float(np.max(np.abs(got["out"][b, h, t] - want)))
        tol = 1e-2 * float(np.max(np.abs(want))) + 2e-3
        assert err <= tol, f"row (b={b}, h={h}, t={t}): max error {err:.3g} > {tol:.3g}"
        worst = max(worst, err)
    for b in range(wl.batch):  # rows at or beyond L_b are not written
        assert np.all(got["out"][b, :, int(lens[b]):] == SENTINEL)
    return worst


def check_codes(wl, inp, got):
    lens = got["lens"]
    want, ys = oracle.encode_cache(inp["K"], inp["W_H"], lens, upto_last=False)
    for b in range(wl.batch):
        Lb = int(lens[b])
        for g in range(wl.n_kv_heads):
            assert_codes_match(got["codes"][b, g, :Lb], want[b, g, :Lb], ys[(b, g)], wl.hash_bits)
            sent = CODE_SENTINEL & (0xFFFF if wl.hash_bits == 16 else 0xFFFFFFFF)
            assert np.all(got["codes"][b, g, Lb:] == sent), "slots beyond L_b must not be written"


SMALL = {
    "ragged_r128": Workload("pf_a", 2, 8, 2, 128, 700, 128, 1, "bf16", seq_len_range=(300, 700)),
    "g1_r32_whole_tiles": Workload("pf_b", 1, 2, 2, 128, 384, 32, 1, "bf16"),
    "g8_r64": Workload("pf_c", 1, 8, 1, 128, 259, 64, 1, "bf16"),
    "r16_ragged": Workload("pf_d", 2, 4, 2, 128, 300, 16, 1, "bf16", seq_len_range=(129, 300)),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_prefill_matches_oracle(H, name):
    wl = SMALL[name]
    inp = make_inputs(wl, seed=71, plant=False)
    Q = _prompt(wl, 71)
    got = run_prefill(H, wl, inp, Q)
    assert got["status"] == 0
    check_rows(wl, inp, Q, got)
    check_codes(wl, inp, got)


def test_prefill_without_codes_and_sharp_softmax(H):
    """codes = NULL gives plain causal attention (same outputs); queries scaled by 4 make
    the row maxima move by more than 2^8 between tiles, so the output is rescaled."""
    wl = Workload("pf_sharp", 1, 8, 2, 128, 1000, 128, 1, "bf16")
    inp = make_inputs(wl, seed=73, plant=False)
    Q = _prompt(wl, 73, q_scale=4.0)
    got = run_prefill(H, wl, inp, Q, with_codes=False)
    assert got["status"] == 0
    check_rows(wl, inp, Q, got)
    got2 = run_prefill(H, wl, inp, Q, with_codes=True)
    assert np.array_equal(got["out"], got2["out"])
    check_codes(wl, inp, got2)


def test_prefill_edge_lengths_and_non_finite_tail(H):
    """L_b of 1, 127, 128, 129 and 0; K/V slots beyond L_b hold NaN and must not reach any output."""
    wl = Workload("pf_edge", 5, 4, 2, 128, 256, 128, 1, "bf16")
    inp = make_inputs(wl, seed=75, plant=False)
    Q = _prompt(wl, 75)
    lens = np.array([1, 127, 128, 129, 0], dtype=np.int32)
    got = run_prefill(H, wl, inp, Q, seq_lens=lens, nan_tail=True)
    assert got["status"] == 0
    assert np.all(np.isfinite(got["out"][0, :, :1]))
    check_rows(wl, inp, Q, got)
    check_codes(wl, inp, got)


def test_prefill_length_beyond_cache_is_flagged(H):
    wl = Workload("pf_over", 1, 2, 1, 128, 200, 32, 1, "bf16")
    inp = make_inputs(wl, seed=77, plant=False)
    Q = _prompt(wl, 77)
    got = run_prefill(H, wl, inp, Q, seq_lens=[201])
    assert got["status"] == 1  # HATA_ERR_INVALID_ARG, clamped to max_seq
    got["lens"] = np.array([200], dtype=np.int32)
    check_rows(wl, inp, Q, got)


def test_prefill_timeout_path(H):
    """The test hook makes the kernel's first bounded wait run out: HATA_ERR_TIMEOUT is
    recorded, the kernel returns, and the next call on a fresh workspace is correct."""
    wl = Workload("pf_to", 1, 4, 2, 128, 300, 32, 1, "bf16")
    inp = make_inputs(wl, seed=79, plant=False)
    Q = _prompt(wl, 79)
    got = run_prefill(H, wl, inp, Q, flags=H.HATA_FLAG_TEST_EXPIRE_WAIT)
    assert got["status"] == 4
    got = run_prefill(H, wl, inp, Q)
    assert got["status"] == 0
    check_rows(wl, inp, Q, got)


def test_prefill_full_size_narrow32(H):
    """The 4 x 65,536-token prompt of the narrow-code workload (32 query / 8 KV heads, r = 32):
    sampled output rows against the oracle, and every key's code against oracle.encode_cache."""
    wl = WORKLOADS["narrow32_b4_64k"]
    inp = make_inputs(wl, seed=0, plant=False)
    d = H.dims_for(wl.batch, wl.n_q_heads, wl.n_kv_heads, 128, wl.hash_bits, wl.max_seq, "bf16")
    Qd = torch.empty((wl.batch, wl.n_q_heads, wl.max_seq, 128), dtype=torch.bfloat16, device="cuda")
    rng = np.random.default_rng(81)
    picks = [(0, 0), (1, 5), (2, 13), (3, 31), (3, 4)]
    rows, qrows = [], {}
    for b in range(wl.batch):
        for h in range(wl.n_q_heads):
            slab = prompt_queries(wl, 0, b, h)
            Qd[b, h] = torch.from_numpy(slab).to("cuda", torch.bfloat16)
            if (b, h) in picks:
                ts = sorted({0, 1, 127, 128, 129, 4095, 30001, wl.max_seq - 1, *rng.integers(0, wl.max_seq, 4).tolist()})
                for t in ts:
                    rows.append((b, h, int(t)))
                    qrows[(b, h, int(t))] = slab[t]
    K, V = dev_float(inp["K"], "bf16"), dev_float(inp["V"], "bf16")
    out = torch.full_like(Qd, SENTINEL)
    codes = dev_codes(np.zeros((wl.batch, wl.n_kv_heads, wl.max_seq, wl.words), dtype=np.uint32))
    ws = torch.zeros(H.hata_prefill_workspace_size(d), dtype=torch.uint8, device="cuda")
    H.hata_prefill_attention(d, Qd, K, V, torch.from_numpy(inp["W_H"]).cuda(), codes,
                             torch.from_numpy(inp["seq_lens"]).cuda(), 0.0, out, ws)
    torch.cuda.synchronize()
    assert H.hata_read_device_status(ws) == 0
    scale = 1.0 / math.sqrt(128)
    for (b, h, t) in rows:
        g = h // wl.group
        want = oracle.prefill_attention_row(qrows[(b, h, t)], inp["K"][b, g], inp["V"][b, g], t, scale)
        gotr = out[b, h, t].float().cpu().numpy()
        err = float(np.max(np.abs(gotr - want)))
        assert err <= 1e-2 * float(np.max(np.abs(want))) + 2e-3, (b, h, t, err)
    del Qd, out
    got_codes = host_codes(codes)
    want, ys = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"], upto_last=False)
    for b in range(wl.batch):
        for g in range(wl.n_kv_heads):
            assert_codes_match(got_codes[b, g], want[b, g], ys[(b, g)], wl.hash_bits)
