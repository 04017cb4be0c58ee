"""CPU oracle for the HATA decode step -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline / reference arm
may import this module.  The product path (the CUDA library and its binding)
never calls it, and it shares no code with that path: it is plain numpy in
float64, written from the method's definitions and kept slow and literal on
purpose so that it can be checked against the pages by eye.

Sources (all from the HATA paper notes, "HATA: Trainable and Hardware-Efficient
Hash-Aware Top-k Attention for Scalable Large Model Inference", ACL 2025):
  * hash function h(x) = 2*Sigmoid(sigma * x W_H) - 1, §方法详解 > 关键设计
    (Learning-to-Hash 建模); at inference the code is its sign, bit-packed
    (§Decode 阶段算法, HashEncode = matrix multiply + Sign + BitPack);
  * Hamming distance = bitcount(bitwise_xor(Q_H, K_H_cache)), §Decode 阶段算法;
  * GQA: scores of the query heads that share one KV cache are aggregated
    (§Decode 阶段算法 and §关键发现 "GQA 兼容"); the aggregate is a sum;
  * top-k select, gather the chosen K/V rows, exact attention on them
    (§Decode 阶段算法; §整体框架 decode phase).
The separate key encoder of decode_step (W_k) follows "HashAttention: Semantic
Sparsity for Faster Inference" (AI summary, Approach: independent key and query
mappings into Hamming space, pivotal tokens by XOR + popcount).

Readings where the pages are silent (each is listed in the design notes):
  * bit j of a code is [y_j > 0] (y = x W_H); bit j lives in 32-bit word j // 32
    at position j % 32 (least significant first);
  * W_H is one [d][r] matrix per KV head, shared by the G query heads of that
    group and by the keys;
  * "top-k" = the k smallest summed distances; ties go to the lower token index;
    the selection is reported in ascending token order; k >= L selects all L;
  * softmax scale defaults to 1/sqrt(d); no sink or recent-window tokens;
  * the new token (slot L_b - 1) is encoded and appended before the scan and is
    a candidate like any other.

Parity pins: every function here is pinned by tests under tests/ marked
"not gpu" (hand-worked golden example, brute force, closed forms, invariants).
The only unpinned quantities are learned-hash quality and speed-ups, which need
trained weights and datasets ("parity unpinned"; not computed here).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "project",
    "sign_bits",
    "pack_bits",
    "unpack_bits",
    "encode",
    "hamming",
    "gqa_scores",
    "topk_select",
    "sparse_attention",
    "decode_step",
    "encode_cache",
    "append_kv",
    "prefill_attention_row",
]


# ----------------------------------------------------------------------------
# HashEncode: projection, sign, bit-pack  (§关键设计 hash function; §Decode 阶段算法)
# ----------------------------------------------------------------------------

def project(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """y = x . W_H in float64.  x: [..., d], W: [d][r] -> y: [..., r]."""
    x64 = np.asarray(x, dtype=np.float64)
    W64 = np.asarray(W, dtype=np.float64)
    return x64 @ W64


def sign_bits(y: np.ndarray) -> np.ndarray:
    """Inference form of h(x): the bit is 1 where y > 0 (the sign of 2*Sigmoid(sigma*y) - 1, sigma > 0)."""
    return np.asarray(y) > 0.0


def pack_bits(bits: np.ndarray) -> np.ndarray:
    """BitPack: bits [..., r] -> uint32 words [..., ceil(r/32)], bit j in word j//32 at position j%32."""
    bits = np.asarray(bits, dtype=bool)
    r = bits.shape[-1]
    n_words = (r + 31) // 32
    words = np.zeros(bits.shape[:-1] + (n_words,), dtype=np.uint32)
    for j in range(r):
        words[..., j // 32] |= bits[..., j].astype(np.uint32) << np.uint32(j % 32)
    return words


def unpack_bits(words: np.ndarray, r: int) -> np.ndarray:
    """Inverse of pack_bits: uint32 words [..., n_words] -> bool bits [..., r]."""
    words = np.asarray(words, dtype=np.uint32)
    bits = np.zeros(words.shape[:-1] + (r,), dtype=bool)
    for j in range(r):
        bits[..., j] = ((words[..., j // 32] >> np.uint32(j % 32)) & np.uint32(1)).astype(bool)
    return bits


def encode(x: np.ndarray, W: np.ndarray):
    """HashEncode of vectors x [..., d] with one W_H [d][r]: returns (codes [..., r/32] uint32, y [..., r] f64)."""
    y = project(x, W)
    return pack_bits(sign_bits(y)), y


def encode_cache(K: np.ndarray, W_H: np.ndarray, seq_lens: np.ndarray, upto_last: bool = True):
    """Prefill encode of a key cache (§整体框架 prefill phase: keys are encoded and their codes cached).

    K: [B][Hkv][Lmax][d]; W_H: [Hkv][d][r].  Encodes slots [0, L_b - 1) when
    upto_last (the decode step appends slot L_b - 1 itself), else [0, L_b).
    Unwritten slots are zero.  Returns (codes [B][Hkv][Lmax][r/32], y list).
    """
    B, Hkv, Lmax, _ = K.shape
    r = W_H.shape[2]
    codes = np.zeros((B, Hkv, Lmax, (r + 31) // 32), dtype=np.uint32)
    ys = {}
    for b in range(B):
        n = int(seq_lens[b]) - (1 if upto_last else 0)
        for g in range(Hkv):
            c, y = encode(K[b, g, :n], W_H[g])
            codes[b, g, :n] = c
            ys[(b, g)] = y
    return codes, ys


def append_kv(K: np.ndarray, V: np.ndarray, new_k: np.ndarray, new_v: np.ndarray, seq_lens: np.ndarray):
    """KV cache update of a decode step (§Decode 阶段算法: the new token's key and value join the cache).

    K, V: [B][Hkv][Lmax][d]; new_k, new_v: [B][Hkv][d].  Returns copies of K and V
    with slot L_b - 1 of every slab of batch b replaced by the new rows, for
    1 <= L_b <= Lmax; other batches are returned unchanged (no slot to write).
    """
    K2, V2 = K.copy(), V.copy()
    Lmax = K.shape[2]
    for b in range(K.shape[0]):
        L = int(seq_lens[b])
        if 1 <= L <= Lmax:
            K2[b, :, L - 1] = new_k[b]
            V2[b, :, L - 1] = new_v[b]
    return K2, V2


# ----------------------------------------------------------------------------
# Hamming distance and the GQA sum  (§Decode 阶段算法; §关键发现 GQA 兼容)
# ----------------------------------------------------------------------------

def hamming(a: np.ndarray, b: np.ndarray, r: int) -> np.ndarray:
    """Hamming distance between packed r-bit codes, by counting differing bits one position at a time."""
    ba = unpack_bits(a, r)
    bb = unpack_bits(b, r)
    return np.sum(ba != bb, axis=-1).astype(np.int64)


def gqa_scores(qcodes: np.ndarray, codes: np.ndarray, r: int) -> np.ndarray:
    """D[t] = sum over the G query heads of Hamming(qcode_h, code_t).

    qcodes: [G][n_words] (the query heads of one KV group); codes: [L][n_words].
    """
    D = np.zeros(codes.shape[0], dtype=np.int64)
    kb = unpack_bits(codes, r)  # [L][r]
    for h in range(qcodes.shape[0]):
        qb = unpack_bits(qcodes[h], r)  # [r]
        D += np.sum(kb != qb[None, :], axis=-1)
    return D


# ----------------------------------------------------------------------------
# Top-k select  (§Decode 阶段算法: select top-k by Hamming distance)
# ----------------------------------------------------------------------------

def topk_select(D: np.ndarray, k: int) -> np.ndarray:
    """The min(k, L) tokens with the smallest distance; ties to the lower index; ascending order."""
    D = np.asarray(D)
    L = D.shape[0]
    t = np.arange(L)
    order = np.lexsort((t, D))  # primary key D, secondary key t
    return np.sort(order[: min(k, L)]).astype(np.int64)


# ----------------------------------------------------------------------------
# Gather + exact attention on the selected rows  (§Decode 阶段算法; §整体框架)
# ----------------------------------------------------------------------------

def sparse_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, S: np.ndarray, scale: float) -> np.ndarray:
    """o_h = softmax_t(scale * q_h . K_t) V over t in S, in float64.  q: [G][d], K/V: [L][d]."""
    Ks = np.asarray(K, dtype=np.float64)[S]
    Vs = np.asarray(V, dtype=np.float64)[S]
    q64 = np.asarray(q, dtype=np.float64)
    out = np.zeros(q64.shape, dtype=np.float64)
    for h in range(q64.shape[0]):
        s = scale * (Ks @ q64[h])
        m = np.max(s)
        p = np.exp(s - m)
        out[h] = (p @ Vs) / np.sum(p)
    return out


# ----------------------------------------------------------------------------
# Prefill attention  (§整体框架 prefill phase: full attention over the prompt,
# during which every key is encoded and its code cached)
# ----------------------------------------------------------------------------

def prefill_attention_row(q_t: np.ndarray, K: np.ndarray, V: np.ndarray, t: int, scale: float) -> np.ndarray:
    """Causal attention output of prompt position t for one query head, in float64:
    o = sum_{s <= t} softmax_s(scale * q_t . K_s) V_s, with K/V the head's KV group
    ([L][d], L > t).  Written out directly from the definition; the prefill of a
    whole prompt is this row for every position t < L_b and every query head h
    (KV group h // G)."""
    q64 = np.asarray(q_t, dtype=np.float64)
    Ks = np.asarray(K[: t + 1], dtype=np.float64)
    Vs = np.asarray(V[: t + 1], dtype=np.float64)
    logits = scale * (Ks @ q64)
    w = np.exp(logits - np.max(logits))
    return (w / np.sum(w)) @ Vs


# ----------------------------------------------------------------------------
# The decode step: encode q, encode + append the new key, scan, select, attend
# ----------------------------------------------------------------------------

def decode_step(q, K, V, W_H, codes, seq_lens, k: int, scale: float | None = None, W_k=None):
    """One HATA decode step over a batch.

    q: [B][Hq][d]; K, V: [B][Hkv][Lmax][d] with the new token already at slot
    L_b - 1; W_H: [Hkv][d][r]; codes: [B][Hkv][Lmax][r/32] holding the codes of
    slots [0, L_b - 1); seq_lens: [B].  W_k (optional, [Hkv][d][r]) is a separate
    key encoder, the form of "HashAttention: Semantic Sparsity for Faster
    Inference" (independent query and key mappings, summary > Approach): the
    queries are encoded with W_H, the new key with W_k, and `codes` must hold
    keys encoded with W_k.  Without it W_H encodes both (HATA).

    Returns a dict with qcode [B][Hq][W], codes (copy with slot L_b - 1 written),
    y_q / y_k (projections, for the sign-exemption band), D (list over (b, g) of
    int arrays of length L_b), idx [B][Hkv][k] (ascending, -1 padded),
    n_sel [B], out [B][Hq][d] float64.
    """
    B, Hq, d = q.shape
    Hkv = K.shape[1]
    r = W_H.shape[2]
    G = Hq // Hkv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    codes = np.array(codes, dtype=np.uint32, copy=True)
    n_words = codes.shape[-1]
    qcode = np.zeros((B, Hq, n_words), dtype=np.uint32)
    y_q = np.zeros((B, Hq, r))
    y_k = np.zeros((B, Hkv, r))
    idx = np.full((B, Hkv, k), -1, dtype=np.int64)
    n_sel = np.zeros(B, dtype=np.int64)
    out = np.zeros((B, Hq, d))
    D_all = {}
    for b in range(B):
        Lb = int(seq_lens[b])
        n_sel[b] = min(k, Lb)
        for g in range(Hkv):
            heads = range(g * G, (g + 1) * G)
            for h in heads:
                qcode[b, h], y_q[b, h] = encode(q[b, h], W_H[g])
            codes[b, g, Lb - 1], y_k[b, g] = encode(K[b, g, Lb - 1], (W_H if W_k is None else W_k)[g])
            D = gqa_scores(qcode[b, g * G : (g + 1) * G], codes[b, g, :Lb], r)
            S = topk_select(D, k)
            idx[b, g, : len(S)] = S
            out[b, g * G : (g + 1) * G] = sparse_attention(q[b, g * G : (g + 1) * G], K[b, g], V[b, g], S, scale)
            D_all[(b, g)] = D
    return {
        "qcode": qcode,
        "codes": codes,
        "y_q": y_q,
        "y_k": y_k,
        "D": D_all,
        "idx": idx,
        "n_sel": n_sel,
        "out": out,
    }
