"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
library through its binding, and compare against the CPU oracle.

Tolerances (from the method's stated correctness targets):
  * codes: bit-exact wherever the oracle's |x . W_H| > 1e-4; sign flips are
    allowed only inside that band (the GPU projects in fp32, the oracle in fp64);
  * Hamming scores and top-k indices: bit-exact given identical codes;
  * attention output: max-abs 2e-2 for bf16, 1e-4 for fp32.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

BAND = 1e-4
TOL = {"bf16": 2e-2, "f32": 1e-4}


def dev_float(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def dev_codes(a: np.ndarray, r: int = 32) -> torch.Tensor:
    """Oracle-packed codes (uint32 words, [..., r/32]) as the library's code tensor: int32 words, or for
    r = 16 one int16 code per token (the word dimension dropped)."""
    a = np.ascontiguousarray(a, dtype=np.uint32)
    if r == 16:
        return torch.from_numpy(np.ascontiguousarray(a[..., 0].astype(np.uint16).view(np.int16))).cuda()
    return torch.from_numpy(a.view(np.int32)).cuda()


def host_codes(t: torch.Tensor) -> np.ndarray:
    """The library's code tensor in the oracle's packing (uint32 words; a 16-bit code in the low half)."""
    a = t.cpu().numpy()
    if a.dtype == np.int16:
        return a.view(np.uint16).astype(np.uint32)[..., None]
    return a.view(np.uint32)


def new_workspace(dims, k) -> torch.Tensor:
    import hash_aware_top_b200 as H

    ws = torch.empty(H.hata_workspace_size(dims, k), dtype=torch.uint8, device="cuda")
    H.hata_workspace_init(ws)
    return ws


def band_mask(y: np.ndarray, r: int) -> np.ndarray:
    """Packed mask of the bits whose projection lies outside the exemption band."""
    return oracle.pack_bits(np.abs(y) > BAND)


def assert_codes_match(gpu: np.ndarray, want: np.ndarray, y: np.ndarray, r: int) -> int:
    """Assert equality outside the band; return how many in-band bits differ."""
    mask = band_mask(y, r)
    diff = (gpu ^ want) & mask
    bad = np.argwhere(diff != 0)
    assert bad.size == 0, f"{len(bad)} code words differ outside the |y| <= {BAND} band, first at {bad[:5].tolist()}"
    return int(sum(bin(int(v)).count("1") for v in np.ravel(gpu ^ want)))


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64)))) if np.size(a) else 0.0


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def run_step(H, wl, inp, codes0, ws=None, with_debug=True, flags=0):
    """One hata_decode_step through the C ABI on the workload's inputs, with the cache holding codes0."""
    d = H.dims_for(wl.batch, wl.n_q_heads, wl.n_kv_heads, 128, wl.hash_bits, wl.max_seq, wl.dtype, flags)
    ws = ws if ws is not None else new_workspace(d, wl.k)
    codes = dev_codes(codes0, wl.hash_bits)
    out = torch.full((wl.batch, wl.n_q_heads, 128), float("nan"), dtype=d.torch_dtype, device="cuda")
    cdt = torch.int16 if wl.hash_bits == 16 else torch.int32
    qcode = torch.zeros(d.code_shape(wl.batch, wl.n_q_heads), dtype=cdt, device="cuda") if with_debug else None
    idx = torch.full((wl.batch, wl.n_kv_heads, wl.k), -99, dtype=torch.int32, device="cuda") if with_debug else None
    H.hata_decode_step(d, dev_float(inp["q"], wl.dtype), dev_float(inp["K"], wl.dtype), dev_float(inp["V"], wl.dtype),
                       torch.from_numpy(inp["W_H"]).cuda(), codes, torch.from_numpy(inp["seq_lens"]).cuda(), wl.k,
                       0.0, out, qcode, idx, ws)
    torch.cuda.synchronize()
    return {
        "codes": host_codes(codes),
        "out": out.float().cpu().numpy(),
        "qcode": host_codes(qcode) if with_debug else None,
        "idx": idx.cpu().numpy() if with_debug else None,
        "ws": ws,
    }


def check_step(wl, inp, codes0, got, W_k=None):
    """Compare one decode step with the oracle.  Where the GPU's fp32 projection
    lands on the other side of zero inside the exemption band, the downstream
    results are checked for validity against the codes the GPU chose.  W_k: a
    separate key encoder (codes0 then holds keys encoded with it)."""
    ref = oracle.decode_step(inp["q"], inp["K"], inp["V"], inp["W_H"], codes0, inp["seq_lens"], wl.k, W_k=W_k)
    G, r = wl.group, wl.hash_bits
    flips = assert_codes_match(got["qcode"], ref["qcode"], ref["y_q"], r)
    for b in range(wl.batch):
        Lb = int(inp["seq_lens"][b])
        for g in range(wl.n_kv_heads):
            flips += assert_codes_match(got["codes"][b, g, Lb - 1], ref["codes"][b, g, Lb - 1], ref["y_k"][b, g], r)
            assert np.array_equal(got["codes"][b, g, :Lb - 1], codes0[b, g, :Lb - 1])
    tol = TOL[wl.dtype]
    for b in range(wl.batch):
        Lb = int(inp["seq_lens"][b])
        for g in range(wl.n_kv_heads):
            hs = slice(g * G, (g + 1) * G)
            if flips == 0:
                want_idx = ref["idx"][b, g]
                want_out = ref["out"][b, hs]
            else:  # validity: the oracle's own steps applied to the codes the GPU chose
                D = oracle.gqa_scores(got["qcode"][b, hs], got["codes"][b, g, :Lb], r)
                S = oracle.topk_select(D, wl.k)
                want_idx = np.full(wl.k, -1)
                want_idx[:len(S)] = S
                want_out = oracle.sparse_attention(inp["q"][b, hs], inp["K"][b, g], inp["V"][b, g], S,
                                                   1 / math.sqrt(128))
            assert np.array_equal(got["idx"][b, g], want_idx), (b, g)
            err = max_abs(got["out"][b, hs], want_out)
            assert err <= tol, (b, g, err)
    return ref, flips
