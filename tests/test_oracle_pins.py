"""Pins for the CPU oracle: each check comes from the pages' definitions or from
mathematics, never from the oracle itself and never from the CUDA path.

Sources: HATA paper notes ("HATA: Trainable and Hardware-Efficient Hash-Aware
Top-k Attention"), sections 关键设计 (hash function) and Decode 阶段算法 (encode,
append, Hamming, GQA aggregate, top-k, gather + attention); HashAttention AI
summary, key results / baselines (random signed projections as LSH).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from hata_inputs import Workload, make_inputs, random_codes, round_to_bf16

from conftest import GOLDEN



def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _py_popcount_xor(a_words, b_words):
    """Hamming distance of two packed codes through Python integers (independent route)."""
    total = 0
    for a, b in zip(a_words, b_words):
        total += bin(int(a) ^ int(b)).count("1")
    return total


# ----------------------------------------------------------------------------
# Golden, hand-worked example (every stage)
# ----------------------------------------------------------------------------

class TestHandWorkedExample:
    g = _load("hand_worked_decode.json")

    def setup_method(self):
        g = self.g
        self.W = np.array(g["W_H_rows"], dtype=np.float64)  # [d][r]
        self.q = np.array(g["q"], dtype=np.float64)
        self.K = np.array(g["K"], dtype=np.float64)
        self.V = np.array(g["V"], dtype=np.float64)

    def test_projection(self):
        np.testing.assert_array_equal(oracle.project(self.q, self.W), np.array(self.g["q_y"]))

    def test_query_codes(self):
        codes, _ = oracle.encode(self.q, self.W)
        assert codes[:, 0].tolist() == self.g["q_code"]

    def test_key_codes(self):
        codes, _ = oracle.encode(self.K, self.W)
        assert codes[:, 0].tolist() == self.g["K_code"]

    def test_per_head_hamming(self):
        qc = np.array(self.g["q_code"], dtype=np.uint32)[:, None]
        kc = np.array(self.g["K_code"], dtype=np.uint32)[:, None]
        for h in range(2):
            got = oracle.hamming(np.broadcast_to(qc[h], kc.shape), kc, 8)
            assert got.tolist() == self.g["hamming_per_head"][h]

    def test_gqa_sum(self):
        qc = np.array(self.g["q_code"], dtype=np.uint32)[:, None]
        kc = np.array(self.g["K_code"], dtype=np.uint32)[:, None]
        assert oracle.gqa_scores(qc, kc, 8).tolist() == self.g["D"]

    @pytest.mark.parametrize("k", ["1", "2", "3", "5", "6", "9"])
    def test_topk(self, k):
        assert oracle.topk_select(np.array(self.g["D"]), int(k)).tolist() == self.g["topk"][k]

    def test_attention_k2(self):
        scale = math.log(3.0) / 14.0
        S = np.array(self.g["topk"]["2"])
        out = oracle.sparse_attention(self.q, self.K, self.V, S, scale)
        np.testing.assert_allclose(out, np.array(self.g["out_k2"]), rtol=0, atol=1e-12)

    def test_attention_k1(self):
        S = np.array(self.g["topk"]["1"])
        out = oracle.sparse_attention(self.q, self.K, self.V, S, 0.5)
        np.testing.assert_array_equal(out, np.array(self.g["out_k1"]))

    def test_decode_step(self):
        """The full step: slots 0..4 hold prefill codes, slot 5 is encoded and appended by the step."""
        g = self.g
        q = self.q[None]  # [B=1][Hq=2][d]
        K = self.K[None, None]  # [1][Hkv=1][L=6][d]
        V = self.V[None, None]
        W = self.W[None]  # [Hkv][d][r]
        codes = np.zeros((1, 1, 6, 1), dtype=np.uint32)
        codes[0, 0, :5, 0] = g["K_code"][:5]
        seq_lens = np.array([6])
        res = oracle.decode_step(q, K, V, W, codes, seq_lens, 2, math.log(3.0) / 14.0)
        assert res["qcode"][0, :, 0].tolist() == g["q_code"]
        assert res["codes"][0, 0, :, 0].tolist() == g["K_code"]
        assert res["D"][(0, 0)].tolist() == g["D"]
        assert res["idx"][0, 0].tolist() == g["topk"]["2"]
        assert res["n_sel"].tolist() == [2]
        np.testing.assert_allclose(res["out"][0], np.array(g["out_k2"]), rtol=0, atol=1e-12)
        # a budget above L pads with -1 and attends densely over all six rows
        res9 = oracle.decode_step(q, K, V, W, codes, seq_lens, 9, 1.0)
        assert res9["idx"][0, 0].tolist() == [0, 1, 2, 3, 4, 5, -1, -1, -1]
        assert res9["n_sel"].tolist() == [6]


def test_bit_order_two_words():
    g = _load("bit_order_r64.json")
    W = -np.ones((1, 64))
    W[0, g["set_bits"]] = 1.0
    codes, _ = oracle.encode(np.array(g["x"]), W)
    assert codes.tolist() == g["words"]
    bits = oracle.unpack_bits(codes, 64)
    assert np.flatnonzero(bits).tolist() == g["set_bits"]


# ----------------------------------------------------------------------------
# Encode: sign of the trainable hash, antipodal symmetry, SimHash closed form
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("sigma", [0.5, 1.0, 10.0])
def test_code_is_sign_of_trainable_hash(sigma):
    """h(x) = 2*Sigmoid(sigma*x W_H) - 1 (section 关键设计); its sign is the code bit, away from y = 0."""
    rng = np.random.default_rng(11)
    d, r = 16, 32
    x = rng.standard_normal((20, d))
    W = rng.standard_normal((d, r)) / math.sqrt(d)
    codes, y = oracle.encode(x, W)
    bits = oracle.unpack_bits(codes, r)
    for n in range(x.shape[0]):
        for j in range(r):
            yj = math.fsum(float(x[n, i]) * float(W[i, j]) for i in range(d))
            h = 2.0 / (1.0 + math.exp(-sigma * yj)) - 1.0
            if abs(yj) > 1e-9:
                assert bits[n, j] == (h > 0.0)


def test_negated_input_complements_code():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((50, 128))
    W = rng.standard_normal((128, 128)) / math.sqrt(128)
    c1, y = oracle.encode(x, W)
    c2, _ = oracle.encode(-x, W)
    mask = oracle.pack_bits(np.abs(y) > 0)
    assert np.array_equal((c1 ^ c2) & mask, mask)


@pytest.mark.parametrize("theta", [0.3, 1.0, 2.0])
def test_simhash_expected_distance(theta):
    """Random Gaussian W_H is random-hyperplane LSH (the LSH baseline of the HashAttention summary):
    each bit differs with probability theta/pi, so E[Ham] = r*theta/pi (Charikar 2002)."""
    rng = np.random.default_rng(13)
    d, r, n = 128, 128, 4000
    W = rng.standard_normal((d, r)) / math.sqrt(128)
    u = rng.standard_normal((n, d))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    v = rng.standard_normal((n, d))
    v -= np.sum(v * u, axis=1, keepdims=True) * u
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    w = math.cos(theta) * u + math.sin(theta) * v
    cu, _ = oracle.encode(u, W)
    cw, _ = oracle.encode(w, W)
    ham = oracle.hamming(cu, cw, r)
    expect = r * theta / math.pi
    sem = ham.std(ddof=1) / math.sqrt(n)
    assert abs(ham.mean() - expect) < 4 * sem


# ----------------------------------------------------------------------------
# Hamming and the GQA sum
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("r", [16, 32, 64, 128, 256])
def test_hamming_against_integer_popcount(r):
    a = random_codes((300,), r, seed=1)
    b = random_codes((300,), r, seed=2)
    got = oracle.hamming(a, b, r)
    want = [_py_popcount_xor(a[i], b[i]) for i in range(300)]
    assert got.tolist() == want


@pytest.mark.parametrize("r", [16, 32, 128])
def test_hamming_metric_properties(r):
    a = random_codes((64,), r, seed=3)
    b = random_codes((64,), r, seed=4)
    c = random_codes((64,), r, seed=5)
    assert np.all(oracle.hamming(a, a, r) == 0)
    assert np.all(oracle.hamming(a, ~a, r) == r)
    assert np.array_equal(oracle.hamming(a, b, r), oracle.hamming(b, a, r))
    assert np.all(oracle.hamming(a, c, r) <= oracle.hamming(a, b, r) + oracle.hamming(b, c, r))


def test_sixteen_bit_code_packing():
    """A 16-bit code is bits 0..15 of one word, bit j at position j (hand-worked): the sign
    pattern + - + + - - - + (then all -) packs to 0b10001101 = 141; all positive gives 0xFFFF."""
    y = -np.ones(16)
    y[[0, 2, 3, 7]] = 1.0
    assert oracle.pack_bits(oracle.sign_bits(y)).tolist() == [141]
    assert oracle.pack_bits(oracle.sign_bits(np.ones(16))).tolist() == [0xFFFF]
    assert oracle.unpack_bits(np.array([141], dtype=np.uint32), 16).nonzero()[0].tolist() == [0, 2, 3, 7]


def test_hamming_bit_by_bit_brute_force_tiny():
    """r = 32, L <= 64: compare against a per-bit Python loop on integers."""
    a = random_codes((64,), 32, seed=6)[:, 0]
    b = random_codes((64,), 32, seed=7)[:, 0]
    got = oracle.hamming(a[:, None], b[:, None], 32)
    for i in range(64):
        want = sum(((int(a[i]) >> j) & 1) != ((int(b[i]) >> j) & 1) for j in range(32))
        assert got[i] == want


@pytest.mark.parametrize("G,r", [(1, 32), (4, 128), (8, 64), (3, 256), (4, 16)])
def test_gqa_sum_is_sum_of_heads(G, r):
    q = random_codes((G,), r, seed=8)
    k = random_codes((200,), r, seed=9)
    D = oracle.gqa_scores(q, k, r)
    want = [sum(_py_popcount_xor(q[h], k[t]) for h in range(G)) for t in range(200)]
    assert D.tolist() == want
    if G == 1:
        assert np.array_equal(D, oracle.hamming(np.broadcast_to(q[0], k.shape), k, r))


# ----------------------------------------------------------------------------
# Top-k
# ----------------------------------------------------------------------------

def _brute_force_topk(D, k):
    """The unique subset S with |S| = min(k, L) whose every (D, t) precedes every outside (D, t)."""
    L = len(D)
    n = min(k, L)
    found = []
    for S in itertools.combinations(range(L), n):
        inside = [(D[t], t) for t in S]
        outside = [(D[t], t) for t in range(L) if t not in S]
        if not outside or max(inside) < min(outside):
            found.append(list(S))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(12))
def test_topk_exhaustive_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    L = int(rng.integers(1, 10))
    k = int(rng.integers(1, 12))
    D = rng.integers(0, 4, size=L)  # few distinct values: many ties
    assert oracle.topk_select(D, k).tolist() == _brute_force_topk(D.tolist(), k)


def test_topk_all_equal_and_oversized_budget():
    assert oracle.topk_select(np.full(50, 7), 5).tolist() == [0, 1, 2, 3, 4]
    assert oracle.topk_select(np.arange(10)[::-1], 20).tolist() == list(range(10))


def test_topk_lexicographic_property_large():
    rng = np.random.default_rng(5)
    D = rng.integers(0, 513, size=5000)
    S = oracle.topk_select(D, 512)
    inside = set(S.tolist())
    worst_in = max((D[t], t) for t in inside)
    best_out = min((D[t], t) for t in range(5000) if t not in inside)
    assert worst_in < best_out and len(inside) == 512 and np.all(np.diff(S) > 0)


# ----------------------------------------------------------------------------
# Attention
# ----------------------------------------------------------------------------

def _textbook_attention(q, K, V, scale):
    """Dense softmax attention with plain Python loops (no max shift)."""
    L, d = K.shape
    out = []
    for h in range(q.shape[0]):
        w = [math.exp(scale * sum(float(q[h, i]) * float(K[t, i]) for i in range(d))) for t in range(L)]
        z = sum(w)
        out.append([sum(w[t] * float(V[t, i]) for t in range(L)) / z for i in range(d)])
    return np.array(out)


def test_full_budget_equals_dense_attention():
    rng = np.random.default_rng(21)
    G, L, d = 3, 40, 16
    q = rng.standard_normal((G, d))
    K = rng.standard_normal((L, d))
    V = rng.standard_normal((L, d))
    got = oracle.sparse_attention(q, K, V, np.arange(L), 1 / math.sqrt(d))
    np.testing.assert_allclose(got, _textbook_attention(q, K, V, 1 / math.sqrt(d)), rtol=1e-12, atol=1e-12)


def test_single_row_and_identical_rows():
    rng = np.random.default_rng(22)
    q = rng.standard_normal((2, 8))
    K = rng.standard_normal((10, 8))
    V = rng.standard_normal((10, 8))
    np.testing.assert_array_equal(oracle.sparse_attention(q, K, V, np.array([7]), 0.3), np.stack([V[7], V[7]]))
    Vc = np.tile(V[3], (10, 1))
    np.testing.assert_allclose(oracle.sparse_attention(q, K, Vc, np.arange(10), 0.3), np.stack([V[3], V[3]]),
                               rtol=0, atol=1e-14)


def test_output_in_convex_hull_of_selected_rows():
    rng = np.random.default_rng(23)
    q = rng.standard_normal((4, 32)) * 3
    K = rng.standard_normal((100, 32))
    V = rng.standard_normal((100, 32))
    S = np.array([3, 9, 50, 77])
    o = oracle.sparse_attention(q, K, V, S, 1.0)
    assert np.all(o <= V[S].max(axis=0) + 1e-12) and np.all(o >= V[S].min(axis=0) - 1e-12)


# ----------------------------------------------------------------------------
# The decode step end to end, on a small synthetic workload
# ----------------------------------------------------------------------------

def test_decode_step_composes_and_finds_planted_keys():
    wl = Workload("t", 2, 8, 2, 128, 700, 128, 64, "bf16", seq_len_range=(300, 700), n_planted=20)
    inp = make_inputs(wl, seed=3)
    codes, _ = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"])
    res = oracle.decode_step(inp["q"], inp["K"], inp["V"], inp["W_H"], codes, inp["seq_lens"], wl.k)
    G = wl.group
    for b in range(wl.batch):
        Lb = int(inp["seq_lens"][b])
        for g in range(wl.n_kv_heads):
            # the appended code is the encoding of the new key
            c, _ = oracle.encode(inp["K"][b, g, Lb - 1], inp["W_H"][g])
            assert np.array_equal(res["codes"][b, g, Lb - 1], c)
            # slots below L_b - 1 are untouched
            assert np.array_equal(res["codes"][b, g, : Lb - 1], codes[b, g, : Lb - 1])
            S = res["idx"][b, g][res["idx"][b, g] >= 0]
            assert len(S) == min(wl.k, Lb)
            # planted keys are close to the group's queries: most of them are selected (sanity, not parity)
            planted = set(inp["planted"][b * wl.n_kv_heads + g].tolist())
            recall = len(planted & set(S.tolist())) / len(planted)
            assert recall > 0.8
            # output equals the oracle's attention over the selected rows
            o = oracle.sparse_attention(inp["q"][b, g * G:(g + 1) * G], inp["K"][b, g], inp["V"][b, g], S,
                                        1 / math.sqrt(128))
            np.testing.assert_array_equal(res["out"][b, g * G:(g + 1) * G], o)


def test_decode_step_separate_key_encoder():
    """HashAttention form (independent query and key encoders; HashAttention
    summary, Approach).  Pins: (1) with W_k = W_H it is the HATA step exactly;
    (2) with W_k = -W_H every key bit flips (y -> -y, and y = 0 has probability 0
    here), so each head's distance becomes r - Ham and the GQA sum G*r - D: the
    step then selects the min(k, L) tokens with the LARGEST D of the plain step,
    ties to the lower index -- checked by a brute-force sort on (-D, t); (3) the
    appended code is the key's encoding under W_k."""
    wl = Workload("t", 2, 8, 2, 128, 500, 128, 40, "bf16", seq_len_range=(200, 500), n_planted=5)
    inp = make_inputs(wl, seed=5)
    lens = inp["seq_lens"]
    codes, _ = oracle.encode_cache(inp["K"], inp["W_H"], lens)
    plain = oracle.decode_step(inp["q"], inp["K"], inp["V"], inp["W_H"], codes, lens, wl.k)
    same = oracle.decode_step(inp["q"], inp["K"], inp["V"], inp["W_H"], codes, lens, wl.k, W_k=inp["W_H"])
    for key in ("qcode", "codes", "idx", "out"):
        assert np.array_equal(plain[key], same[key]), key
    W_neg = -inp["W_H"]
    codes_neg, _ = oracle.encode_cache(inp["K"], W_neg, lens)
    flip = oracle.decode_step(inp["q"], inp["K"], inp["V"], inp["W_H"], codes_neg, lens, wl.k, W_k=W_neg)
    G, r = wl.group, wl.hash_bits
    assert np.array_equal(flip["qcode"], plain["qcode"])
    for b in range(wl.batch):
        Lb = int(lens[b])
        for g in range(wl.n_kv_heads):
            c, _ = oracle.encode(inp["K"][b, g, Lb - 1], W_neg[g])
            assert np.array_equal(flip["codes"][b, g, Lb - 1], c)
            D = np.asarray(plain["D"][(b, g)])
            assert np.array_equal(np.asarray(flip["D"][(b, g)]), G * r - D)
            want = sorted(sorted(range(Lb), key=lambda t: (-int(D[t]), t))[: min(wl.k, Lb)])
            got = flip["idx"][b, g][flip["idx"][b, g] >= 0]
            assert got.tolist() == want


def test_bf16_rounding_of_inputs():
    """The input generator's bf16 rounding is round-to-nearest-even (checked against torch)."""
    import torch

    x = np.random.default_rng(0).standard_normal(10000).astype(np.float32) * 100
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(round_to_bf16(x), want)


def test_append_kv_writes_only_the_new_slot():
    """The cache update puts the new rows at slot L_b - 1 (the position of the new
    token in a cache of L_b tokens) and nowhere else; L_b outside [1, Lmax] writes nothing."""
    rng = np.random.default_rng(5)
    B, Hkv, Lmax, d = 4, 2, 6, 3
    K = rng.standard_normal((B, Hkv, Lmax, d))
    V = rng.standard_normal((B, Hkv, Lmax, d))
    nk = rng.standard_normal((B, Hkv, d))
    nv = rng.standard_normal((B, Hkv, d))
    lens = np.array([1, 6, 0, 7])
    K2, V2 = oracle.append_kv(K, V, nk, nv, lens)
    for b in range(B):
        for g in range(Hkv):
            for t in range(Lmax):
                hit = 1 <= lens[b] <= Lmax and t == lens[b] - 1
                assert np.array_equal(K2[b, g, t], nk[b, g] if hit else K[b, g, t])
                assert np.array_equal(V2[b, g, t], nv[b, g] if hit else V[b, g, t])
    assert np.array_equal(K2[0, :, 0], nk[0]) and np.array_equal(V2[1, :, 5], nv[1])


def test_prefill_row_closed_forms():
    """Causal prefill attention: position 0 sees only itself (output = V_0 exactly);
    identical keys give the plain mean of the visible values; two positions give
    the two-term softmax written by hand."""
    rng = np.random.default_rng(9)
    d, L = 4, 6
    K = rng.standard_normal((L, d))
    V = rng.standard_normal((L, d))
    q = rng.standard_normal(d)
    assert np.array_equal(oracle.prefill_attention_row(q, K, V, 0, 0.5), V[0])
    Keq = np.tile(K[:1], (L, 1))
    assert np.allclose(oracle.prefill_attention_row(q, Keq, V, 4, 0.5), V[:5].mean(axis=0), atol=1e-15)
    s0, s1 = 0.5 * q @ K[0], 0.5 * q @ K[1]
    want = (math.exp(s0) * V[0] + math.exp(s1) * V[1]) / (math.exp(s0) + math.exp(s1))
    assert np.allclose(oracle.prefill_attention_row(q, K, V, 1, 0.5), want, atol=1e-14)
    # later positions never influence earlier rows
    K2, V2 = K.copy(), V.copy()
    K2[3:] += 100.0
    V2[3:] -= 7.0
    assert np.array_equal(oracle.prefill_attention_row(q, K2, V2, 2, 0.5), oracle.prefill_attention_row(q, K, V, 2, 0.5))


def test_prefill_row_is_sparse_attention_over_the_prefix():
    """Row t of the causal prefill equals attention over the selected set {0..t}
    (the decode step's attention with every earlier token selected)."""
    rng = np.random.default_rng(10)
    d, L = 8, 40
    K = rng.standard_normal((L, d))
    V = rng.standard_normal((L, d))
    q = rng.standard_normal(d)
    for t in (0, 7, 39):
        got = oracle.prefill_attention_row(q, K, V, t, 0.3)
        want = oracle.sparse_attention(q[None, :], K, V, np.arange(t + 1), 0.3)[0]
        assert np.allclose(got, want, atol=1e-12)
