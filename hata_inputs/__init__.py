"""Seeded synthetic inputs for the HATA decode step.

This module only draws random numbers and lays them out. It holds none of the
method's arithmetic (no projection, no sign, no Hamming distance, no top-k, no
attention), so both the CPU oracle's tests and the CUDA path can take their
inputs from it without sharing any of the computation under test.

Workloads follow the decode-speed experiment of the HATA paper notes
("HATA: Trainable and Hardware-Efficient Hash-Aware Top-k Attention", section
推理速度: Llama-3.1-8B at 32K/64K/128K context, 512-token budget from the
LongBench-e table) and the narrow-code setting of "HashAttention: Semantic
Sparsity for Faster Inference" (32-bit signatures, 32x sparsity). No dataset,
prompt or trained weight is used: q, K, V are Gaussian, W_H is a Gaussian
random projection, and a small fraction of keys is planted near the query so
that top-k has something to find.

Recipe (all draws from numpy PCG64 streams spawned from SeedSequence(seed)):
  * q, K, V ~ N(0, 1), rounded to the workload dtype (bf16 round-to-nearest-even
    or fp32).
  * W_H ~ N(0, 1/128) in fp32, one [d][r] matrix per KV head.
  * per-sequence lengths: fixed, or uniform integers in [lo, hi] (ragged batch).
  * planted keys: n_p positions per (batch, KV head), drawn without replacement
    from [0, L_b - 1) (the slot L_b - 1 holds the new token), each overwritten by
    0.8 * qbar_g + 0.6 * N(0, 1) and rounded, where qbar_g is the fp32 mean of
    the G query heads of KV group g.  n_p = 40 for the tiny workload, otherwise
    floor(0.01 * L_b).
  * prefill prompts: queries at every position, [Lmax][d] per (batch, query head)
    ~ N(0, 1) (optionally scaled, for sharper softmax), each slab from its own
    stream so that sampled rows can be redrawn without the rest.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "round_to_bf16",
    "bf16_bits",
    "make_inputs",
    "random_codes",
    "random_scores",
    "random_indices",
    "prompt_queries",
]

N_STREAMS = 8
S_Q, S_K, S_V, S_W, S_LENS, S_PLANT_POS, S_PLANT_NOISE, S_CODES = range(N_STREAMS)
PROMPT_TAG = 0x5071  # spawn key of the prompt queries' streams


@dataclass(frozen=True)
class Workload:
    """Shape and distribution of one synthetic decode workload."""

    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    max_seq: int
    hash_bits: int
    k: int
    dtype: str  # "f32" or "bf16": element type of q, K, V and the output
    seq_len_range: Optional[tuple] = None  # (lo, hi) inclusive; None -> all max_seq
    n_planted: Optional[int] = None  # None -> floor(0.01 * L_b)
    planted_scale: float = 0.8
    noise_scale: float = 0.6

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def words(self) -> int:
        """32-bit words per code in the oracle's packing (a 16-bit code fills the low half of one)."""
        return (self.hash_bits + 31) // 32

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # single-head fp32 decode, 4K context, 40 planted keys
    "tiny_f32_4k": Workload("tiny_f32_4k", 1, 1, 1, 128, 4096, 128, 256, "f32", n_planted=40),
    # Llama-3.1-8B-shaped layer (32 q heads / 8 KV heads, GQA 4), 32K context
    "llama8b_32k": Workload("llama8b_32k", 1, 32, 8, 128, 32768, 128, 512, "bf16"),
    # same layer at 128K context: the long-context roofline case
    "llama8b_128k": Workload("llama8b_128k", 1, 32, 8, 128, 131072, 128, 512, "bf16"),
    # batch 16, ragged lengths in [8192, 65536], budget 1024
    "batch16_ragged": Workload(
        "batch16_ragged", 16, 32, 8, 128, 65536, 128, 1024, "bf16", seq_len_range=(8192, 65536)
    ),
    # HashAttention-style 32-bit codes, batch 4, 64K context, budget seq/32
    "narrow32_b4_64k": Workload("narrow32_b4_64k", 4, 32, 8, 128, 65536, 32, 2048, "bf16"),
}


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32 holding bf16 values."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of fp32 values that are already bf16-representable."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("values are not bf16-representable")
    return (u >> np.uint32(16)).astype(np.uint16)


def _round(a: np.ndarray, dtype: str) -> np.ndarray:
    a = np.asarray(a, dtype=np.float32)
    return round_to_bf16(a) if dtype == "bf16" else a


def _streams(seed: int):
    return [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(N_STREAMS)]


def make_inputs(wl: Workload, seed: int = 0, plant: bool = True) -> dict:
    """Draw one decode step's inputs.

    Returns a dict of numpy arrays (C-contiguous):
      q        [B][Hq][d]         fp32 holding dtype-rounded values
      K, V     [B][Hkv][Lmax][d]  fp32 holding dtype-rounded values; row L_b-1 is the new token
      W_H      [Hkv][d][r]        fp32
      seq_lens [B]                int32, cached length including the new token
      planted  list over (b, g) of int64 position arrays (for recall sanity checks)
    """
    B, Hq, Hkv, d, L, r = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.max_seq, wl.hash_bits
    if Hq % Hkv:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    rs = _streams(seed)
    q = _round(rs[S_Q].standard_normal((B, Hq, d), dtype=np.float32), wl.dtype)
    K = _round(rs[S_K].standard_normal((B, Hkv, L, d), dtype=np.float32), wl.dtype)
    V = _round(rs[S_V].standard_normal((B, Hkv, L, d), dtype=np.float32), wl.dtype)
    W = (rs[S_W].standard_normal((Hkv, d, r), dtype=np.float32) * np.float32(1.0 / np.sqrt(128.0))).astype(
        np.float32
    )
    if wl.seq_len_range is None:
        seq_lens = np.full(B, L, dtype=np.int32)
    else:
        lo, hi = wl.seq_len_range
        seq_lens = rs[S_LENS].integers(lo, hi, size=B, endpoint=True).astype(np.int32)
        if seq_lens.max() > L:
            raise ValueError("seq_len_range exceeds max_seq")
    planted = []
    G = wl.group
    for b in range(B):
        Lb = int(seq_lens[b])
        for g in range(Hkv):
            if not plant or Lb < 2:
                planted.append(np.zeros(0, dtype=np.int64))
                continue
            n_p = wl.n_planted if wl.n_planted is not None else int(0.01 * Lb)
            n_p = min(n_p, Lb - 1)
            pos = np.sort(rs[S_PLANT_POS].choice(Lb - 1, size=n_p, replace=False)).astype(np.int64)
            qbar = q[b, g * G : (g + 1) * G].astype(np.float32).mean(axis=0, dtype=np.float32)
            noise = rs[S_PLANT_NOISE].standard_normal((n_p, d), dtype=np.float32)
            K[b, g, pos] = _round(
                np.float32(wl.planted_scale) * qbar[None, :] + np.float32(wl.noise_scale) * noise, wl.dtype
            )
            planted.append(pos)
    return {"q": q, "K": K, "V": V, "W_H": W, "seq_lens": seq_lens, "planted": planted}


def prompt_queries(wl: Workload, seed: int, b: int, h: int, q_scale: float = 1.0) -> np.ndarray:
    """The prefill prompt's queries of batch b, query head h: [Lmax][d] ~ N(0, q_scale^2),
    rounded to the workload dtype.  Each (b, h) slab has its own stream (SeedSequence
    of (seed, PROMPT_TAG, b, h)), so a slab can be drawn again without the rest."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, PROMPT_TAG, b, h]))
    x = rng.standard_normal((wl.max_seq, wl.head_dim), dtype=np.float32)
    return _round(x * np.float32(q_scale), wl.dtype)


def random_codes(shape, hash_bits: int, seed: int = 0) -> np.ndarray:
    """Uniformly random packed codes: uint32 array of shape (*shape, ceil(hash_bits / 32)); a 16-bit code
    occupies the low half of its one word."""
    rng = _streams(seed)[S_CODES]
    top = 2 ** min(hash_bits, 32)
    return rng.integers(0, top, size=tuple(shape) + ((hash_bits + 31) // 32,), dtype=np.uint64).astype(np.uint32)


def random_scores(shape, max_value: int, seed: int = 0, n_distinct: Optional[int] = None) -> np.ndarray:
    """Integer scores in [0, max_value] (int32); with n_distinct, drawn from that many values (heavy ties)."""
    rng = _streams(seed)[S_CODES]
    if n_distinct is None:
        return rng.integers(0, max_value, size=shape, endpoint=True).astype(np.int32)
    vals = rng.choice(max_value + 1, size=min(n_distinct, max_value + 1), replace=False)
    return vals[rng.integers(0, len(vals), size=shape)].astype(np.int32)


def random_indices(n_units: int, L: np.ndarray, k: int, seed: int = 0) -> np.ndarray:
    """Per unit, min(k, L_u) distinct ascending indices below L_u, -1 padded to k (int32 [n_units][k])."""
    rng = _streams(seed)[S_CODES]
    out = np.full((n_units, k), -1, dtype=np.int32)
    for u in range(n_units):
        n = min(k, int(L[u]))
        if n > 0:
            out[u, :n] = np.sort(rng.choice(int(L[u]), size=n, replace=False))
    return out
