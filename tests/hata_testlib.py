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


def dev_codes(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint32).view(np.int32)).cuda()


def host_codes(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


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
