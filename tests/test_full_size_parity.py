"""Oracle parity of the decode step at the full size of every benchmark workload.

Each case runs hata_decode_step through the C ABI on the exact inputs the
benchmark times (same workload definition, seed 0, planted keys as generated)
and compares every (batch, KV head) unit element by element with the CPU
oracle: the query codes and the appended key code outside the 1e-4 band, the
top-k indices bit for bit, the outputs within the dtype tolerance.  At 128K
context the selection threshold falls inside the cluster of planted keys
(1,310 planted per unit against a budget of 512), so ties at the threshold are
split across the slices that different thread blocks score.

The narrow-code workload's prefill (every key of a 4 x 8 x 65,536 cache encoded
at r = 32) is compared with the oracle's encode as well.
"""
import numpy as np
import pytest

import oracle
from hata_inputs import WORKLOADS, make_inputs

from hata_testlib import assert_codes_match, check_step, dev_codes, dev_float, host_codes, new_workspace, run_step

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def H():
    import hash_aware_top_b200 as H

    return H


_CACHE = {}


def _inputs(name):
    if name not in _CACHE:
        _CACHE.clear()  # one workload's host arrays at a time (batch16_ragged holds ~9 GB)
        wl = WORKLOADS[name]
        inp = make_inputs(wl, seed=0)
        codes0, _ = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"])
        _CACHE[name] = (wl, inp, codes0)
    return _CACHE[name]


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_decode_step_full_size(H, name):
    wl, inp, codes0 = _inputs(name)
    got = run_step(H, wl, inp, codes0)
    check_step(wl, inp, codes0, got)
    assert H.hata_read_device_status(got["ws"]) == 0


@pytest.mark.parametrize("flags", [1, 4, 5])
def test_decode_step_full_size_other_launch_forms(H, flags):
    """The headline shape with early prefetch (codes streamed before the preceding
    kernel finishes), in the all-SM form, and both: the same results."""
    wl, inp, codes0 = _inputs("llama8b_128k")
    got = run_step(H, wl, inp, codes0, flags=flags)
    check_step(wl, inp, codes0, got)
    assert H.hata_read_device_status(got["ws"]) == 0


def test_prefill_encode_full_size_narrow32(H):
    """hata_encode_append over every key of the 4 x 8 x 65,536 narrow-code cache (r = 32)."""
    wl = WORKLOADS["narrow32_b4_64k"]
    _CACHE.clear()
    inp = make_inputs(wl, seed=0)
    d = H.dims_for(wl.batch, wl.n_q_heads, wl.n_kv_heads, 128, wl.hash_bits, wl.max_seq, wl.dtype)
    codes = dev_codes(np.zeros((wl.batch, wl.n_kv_heads, wl.max_seq, wl.words), dtype=np.uint32))
    ws = new_workspace(d, wl.k)
    H.hata_encode_append(d, dev_float(inp["K"], wl.dtype), wl.n_kv_heads, wl.max_seq, wl.max_seq,
                         torch.from_numpy(inp["seq_lens"]).cuda(), torch.from_numpy(inp["W_H"]).cuda(), codes,
                         wl.max_seq, ws)
    got = host_codes(codes)
    assert H.hata_read_device_status(ws) == 0
    want, ys = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"], upto_last=False)
    for b in range(wl.batch):
        for g in range(wl.n_kv_heads):
            assert_codes_match(got[b, g], want[b, g], ys[(b, g)], wl.hash_bits)
