"""The decode step's timeout path, made to run on purpose and without a GPU fault.

With the HATA_FLAG_TEST_EXPIRE_WAIT launch flag the step's first bounded wait is
made on a barrier that nothing completes, with a short limit.  It has to run out,
record HATA_ERR_TIMEOUT in the workspace's status word, skip the remaining work
(every thread block still reaches its cluster barriers, and its own copies land
before it exits), and leave the GPU usable: the next normal call on a
re-initialised workspace matches the oracle.
"""
import numpy as np
import pytest

import oracle
from hata_inputs import Workload, make_inputs

from hata_testlib import check_step, new_workspace, run_step

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def H():
    import hash_aware_top_b200 as H

    return H


@pytest.mark.parametrize("wl", [
    Workload("t_llama", 1, 32, 8, 128, 40000, 128, 512, "bf16"),
    Workload("t_ragged", 3, 8, 2, 128, 9000, 64, 300, "f32", seq_len_range=(1, 9000)),
])
def test_expired_wait_reports_timeout_then_recovers(H, wl):
    inp = make_inputs(wl, seed=31)
    codes0, _ = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"])
    got = run_step(H, wl, inp, codes0, flags=H.HATA_FLAG_TEST_EXPIRE_WAIT)
    ws = got["ws"]
    assert H.hata_read_device_status(ws) == H.HATA_ERR_TIMEOUT
    assert H.hata_read_device_status(ws) == 0  # the read cleared it
    H.hata_workspace_init(ws)
    again = run_step(H, wl, inp, codes0, ws=ws)
    check_step(wl, inp, codes0, again)
    assert H.hata_read_device_status(ws) == 0


def test_expired_wait_on_a_paged_cache(H):
    wl = Workload("t_paged", 2, 8, 2, 128, 4096, 128, 200, "bf16")
    inp = make_inputs(wl, seed=33)
    d = H.dims_for(wl.batch, wl.n_q_heads, wl.n_kv_heads, 128, 128, wl.max_seq, "bf16",
                   H.HATA_FLAG_TEST_EXPIRE_WAIT)
    bs, nb = 256, 2 * 16
    ws = new_workspace(d, wl.k)
    K = torch.zeros((nb, 2, bs, 128), dtype=torch.bfloat16, device="cuda")
    V = torch.zeros_like(K)
    codes = torch.zeros((nb, 2, bs, 4), dtype=torch.int32, device="cuda")
    btab = torch.arange(nb, dtype=torch.int32, device="cuda").reshape(2, 16)
    out = torch.empty((2, 8, 128), dtype=torch.bfloat16, device="cuda")
    W = torch.from_numpy(inp["W_H"]).cuda()
    H.hata_decode_step_paged(d, torch.from_numpy(inp["q"]).cuda().bfloat16(), K, V, W, W, codes, btab, bs,
                             torch.from_numpy(inp["seq_lens"]).cuda(), wl.k, 0.0, out, None, None, ws)
    assert H.hata_read_device_status(ws) == H.HATA_ERR_TIMEOUT
