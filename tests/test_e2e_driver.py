"""The benchmark's end-to-end loop (hash_aware_top_b200/libhata_e2e.so) calls the public
C ABI with its inputs copied from pinned host memory each step: after it, the caches hold
the new K/V rows at slot L_b - 1 and the pinned output equals a direct hata_decode_step
on the updated buffers."""
import ctypes
import os

import numpy as np
import pytest

import oracle
from hata_inputs import Workload, make_inputs

from hata_testlib import dev_codes, dev_float, new_workspace

torch = pytest.importorskip("torch")


def _e2e_lib():
    import hash_aware_top_b200 as H

    return ctypes.CDLL(os.path.join(os.path.dirname(H.LIB_PATH), "libhata_e2e.so"))


def test_e2e_library_exports_its_loop():
    assert hasattr(_e2e_lib(), "hata_e2e_run")


@pytest.mark.gpu
@pytest.mark.parametrize("flags", [0, 4])
def test_e2e_loop_matches_a_direct_call(flags):
    import bench
    import hash_aware_top_b200 as H

    wl = Workload("e2e", 2, 8, 2, 128, 3000, 128, 64, "bf16", seq_len_range=(1000, 3000))
    inp = make_inputs(wl, seed=61)
    codes0, _ = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"])
    d = H.dims_for(wl.batch, wl.n_q_heads, wl.n_kv_heads, 128, 128, wl.max_seq, "bf16", flags)
    ws = new_workspace(d, wl.k)
    lay = {"q": dev_float(inp["q"], "bf16"), "K": dev_float(inp["K"], "bf16"), "V": dev_float(inp["V"], "bf16"),
           "W": torch.from_numpy(inp["W_H"]).cuda(), "codes": dev_codes(codes0),
           "lens": torch.from_numpy(inp["seq_lens"]).cuda(),
           "out": torch.empty((wl.batch, wl.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")}
    in_host, out_host = bench.e2e_inputs(wl, lay, inp["seq_lens"])
    # new K/V rows that differ from the cached ones
    nq = wl.batch * wl.n_q_heads
    rng = np.random.default_rng(3)
    in_host[nq:] = torch.from_numpy(rng.standard_normal((in_host.shape[0] - nq, 128)).astype(np.float32)).bfloat16()
    stage = torch.empty_like(in_host, device="cuda")
    stream = torch.cuda.Stream()
    dms, hms = bench.run_e2e(H, d, wl.k, 3, [lay], [stage], in_host, out_host, ws, stream)
    assert dms > 0 and hms > 0
    torch.cuda.synchronize()
    nk = in_host[nq:nq + wl.batch * wl.n_kv_heads].reshape(wl.batch, wl.n_kv_heads, 128)
    nv = in_host[nq + wl.batch * wl.n_kv_heads:].reshape(wl.batch, wl.n_kv_heads, 128)
    for b in range(wl.batch):
        L = int(inp["seq_lens"][b])
        assert torch.equal(lay["K"][b, :, L - 1].cpu(), nk[b]) and torch.equal(lay["V"][b, :, L - 1].cpu(), nv[b])
    ref = torch.empty_like(lay["out"])
    H.hata_decode_step(d, lay["q"], lay["K"], lay["V"], lay["W"], lay["codes"], lay["lens"], wl.k, 0.0, ref, None,
                       None, ws)
    torch.cuda.synchronize()
    assert torch.equal(out_host, ref.cpu())
    assert H.hata_read_device_status(ws) == 0
