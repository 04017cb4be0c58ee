"""CPU checks of the C ABI: the library loads, exports every symbol that
include/hata.h declares, and rejects bad arguments on the host before any
launch.  No call here reaches a kernel."""
import ctypes
import os
import re

import pytest

from conftest import ROOT


@pytest.fixture(scope="module")
def H():
    import hash_aware_top_b200 as H

    return H


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "hata.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"HATA_API\s+[\w\s\*]*?\b(hata_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared_symbols()
    for n in ("hata_encode_append", "hata_hamming_scores", "hata_topk", "hata_sparse_decode", "hata_decode_step"):
        assert n in names


def test_library_exports_every_declared_symbol(H):
    lib = ctypes.CDLL(H.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert set(_declared_symbols()) <= set(H.EXPORTED_SYMBOLS) | {"hata_workspace_size"}


def test_version_and_status_strings(H):
    assert H.hata_version() >= 100
    assert H.hata_status_string(0) == "ok"
    assert "timed out" in H.hata_status_string(4)
    assert H.hata_status_string(99) == "unknown status"


@pytest.mark.parametrize(
    "dims,status",
    [
        ((1, 32, 8, 128, 128, 1024, 1), 0),
        ((0, 32, 8, 128, 128, 1024, 1), 1),  # batch
        ((1, 30, 8, 128, 128, 1024, 1), 1),  # Hq not a multiple of Hkv
        ((1, 32, 8, 64, 128, 1024, 1), 2),  # head_dim
        ((1, 32, 8, 128, 96, 1024, 1), 2),  # hash_bits
        ((1, 32, 8, 128, 128, 0, 1), 1),  # max_seq
        ((1, 32, 8, 128, 128, 1024, 7), 1),  # dtype
        ((1, 64, 2, 128, 128, 1024, 1), 2),  # group of 32 heads
    ],
)
def test_workspace_size_validates_dims(H, dims, status):
    d = H.Dims(*dims, 0)
    n = ctypes.c_size_t(0)
    assert H.lib.hata_workspace_size(ctypes.byref(d), 512, ctypes.byref(n)) == status
    if status == 0:
        assert n.value > 0


def test_workspace_size_grows_with_context(H):
    a = H.hata_workspace_size(H.dims_for(1, 32, 8, 128, 128, 32768, "bf16"), 512)
    b = H.hata_workspace_size(H.dims_for(1, 32, 8, 128, 128, 131072, "bf16"), 512)
    assert b > a


def test_calls_reject_bad_arguments_before_launch(H):
    d = H.dims_for(1, 4, 1, 128, 128, 64, "bf16")
    P = ctypes.c_void_p
    fake = P(0x1000)  # never dereferenced: every call below must fail validation first
    null = P(0)
    lib = H.lib
    # null pointers
    assert lib.hata_encode_append(ctypes.byref(d), null, 1, 64, 1, null, fake, fake, 64, fake, 16, null) == 1
    # the encode's status workspace: missing, misaligned or smaller than one status word
    assert lib.hata_encode_append(ctypes.byref(d), fake, 1, 64, 1, null, fake, fake, 64, null, 16, null) == 5
    assert lib.hata_encode_append(ctypes.byref(d), fake, 1, 64, 1, null, fake, fake, 64, P(0x1008), 16, null) == 5
    assert lib.hata_encode_append(ctypes.byref(d), fake, 1, 64, 1, null, fake, fake, 64, fake, 8, null) == 5
    assert lib.hata_hamming_scores(ctypes.byref(d), fake, fake, null, fake, null) == 1
    # prefill attention: bf16 only, pointers required, scale >= 0, workspace large enough
    F0 = ctypes.c_float(0.0)
    pf = lambda dd, q, codes, W, scale, ws, wsb: lib.hata_prefill_attention(  # noqa: E731
        ctypes.byref(dd), q, fake, fake, W, codes, fake, scale, fake, ws, wsb, null)
    db = H.dims_for(1, 4, 1, 128, 32, 64, "bf16")
    assert pf(H.dims_for(1, 4, 1, 128, 32, 64, "f32"), fake, fake, fake, F0, fake, 1 << 30) == 2
    assert pf(db, null, fake, fake, F0, fake, 1 << 30) == 1
    assert pf(db, fake, fake, null, F0, fake, 1 << 30) == 1  # codes without W_H
    assert pf(db, fake, fake, fake, ctypes.c_float(-1.0), fake, 1 << 30) == 1
    assert pf(db, fake, fake, fake, F0, fake, 16) == 5
    assert pf(db, fake, fake, fake, F0, null, 1 << 30) == 5
    n = ctypes.c_size_t(0)
    assert lib.hata_prefill_workspace_size(ctypes.byref(db), ctypes.byref(n)) == 0 and n.value >= 16 + 3 * 32 * 256
    # the cache update: every pointer required, all 16-byte aligned
    assert lib.hata_append_kv(ctypes.byref(d), fake, fake, fake, fake, null, null) == 1
    assert lib.hata_append_kv(ctypes.byref(d), null, fake, fake, fake, fake, null) == 1
    assert lib.hata_append_kv(ctypes.byref(d), fake, fake, P(0x1008), fake, fake, null) == 1
    # the paged cache update: pointers, alignment, a power-of-two block size in [16, 65536], a pool
    assert lib.hata_append_kv_paged(ctypes.byref(d), fake, fake, fake, fake, null, 64, 4, fake, null) == 1
    assert lib.hata_append_kv_paged(ctypes.byref(d), fake, fake, fake, fake, fake, 48, 4, fake, null) == 1
    assert lib.hata_append_kv_paged(ctypes.byref(d), fake, fake, fake, fake, fake, 64, 0, fake, null) == 1
    assert lib.hata_append_kv_paged(ctypes.byref(d), fake, P(0x1004), fake, fake, fake, 64, 4, fake, null) == 1
    # k < 1
    assert lib.hata_topk(ctypes.byref(d), fake, fake, 0, fake, null, fake, 1 << 20, null) == 1
    # workspace too small / missing
    assert lib.hata_topk(ctypes.byref(d), fake, fake, 4, fake, null, fake, 16, null) == 5
    assert lib.hata_sparse_decode(ctypes.byref(d), fake, fake, fake, fake, 4, ctypes.c_float(0.0), fake, null,
                                  1 << 30, null) == 5
    # misaligned pointers
    odd = P(0x1001)
    assert lib.hata_decode_step(ctypes.byref(d), odd, fake, fake, fake, fake, fake, 4, ctypes.c_float(0.0), fake,
                                null, null, fake, 1 << 30, null) == 1
    # non-finite scale
    assert lib.hata_sparse_decode(ctypes.byref(d), fake, fake, fake, fake, 4, ctypes.c_float(float("nan")), fake,
                                  fake, 1 << 30, null) == 1
    # x_heads not a multiple of Hkv, unsupported dims
    d2 = H.dims_for(1, 4, 2, 128, 128, 64, "bf16")
    assert lib.hata_encode_append(ctypes.byref(d2), fake, 3, 64, 1, null, fake, fake, 64, fake, 16, null) == 1
    d3 = H.dims_for(1, 4, 1, 128, 100, 64, "bf16")
    assert lib.hata_hamming_scores(ctypes.byref(d3), fake, fake, fake, fake, null) == 2
    assert lib.hata_read_device_status(null, null, ctypes.byref(ctypes.c_int())) == 1


def test_separate_encoder_and_paged_calls_reject_bad_arguments(H):
    """hata_decode_step_qk and hata_decode_step_paged validate on the host: missing or
    misaligned matrices and tables, block sizes that are not a power of two in
    [16, 65536], an empty pool."""
    d = H.dims_for(1, 4, 1, 128, 128, 1024, "bf16")
    P = ctypes.c_void_p
    fake, odd, null = P(0x1000), P(0x1008), P(0)
    lib = H.lib
    f0 = ctypes.c_float(0.0)
    # qk: W_k missing / misaligned
    assert lib.hata_decode_step_qk(ctypes.byref(d), fake, fake, fake, fake, null, fake, fake, 4, f0, fake, null,
                                   null, fake, 1 << 30, null) == 1
    assert lib.hata_decode_step_qk(ctypes.byref(d), fake, fake, fake, fake, odd, fake, fake, 4, f0, fake, null,
                                   null, fake, 1 << 30, null) == 1

    def paged(block_table, bs, n_blocks, k=4):
        return lib.hata_decode_step_paged(ctypes.byref(d), fake, fake, fake, fake, fake, fake, block_table, bs,
                                          n_blocks, fake, k, f0, fake, null, null, fake, 1 << 30, null)

    assert paged(null, 64, 16) == 1          # no block table
    for bs in (0, 8, 15, 24, 100, 1 << 17):  # not a power of two in [16, 65536]
        assert paged(fake, bs, 16) == 1, bs
    assert paged(fake, 64, 0) == 1           # empty pool
    assert paged(fake, 64, 16, k=0) == 1     # k < 1


def test_binding_refuses_cpu_tensors(H):
    import torch

    d = H.dims_for(1, 4, 1, 128, 128, 64, "bf16")
    with pytest.raises(ValueError, match="CUDA tensor"):
        H.hata_hamming_scores(d, torch.zeros(1, 4, 4, dtype=torch.int32), torch.zeros(1, 1, 64, 4, dtype=torch.int32),
                              torch.zeros(1, dtype=torch.int32), torch.zeros(1, 1, 64, dtype=torch.int32))


def test_unknown_flags_rejected(H):
    n = ctypes.c_size_t(0)
    d = H.dims_for(1, 32, 8, 128, 128, 1024, "bf16", flags=H.HATA_FLAG_EARLY_PREFETCH)
    assert H.lib.hata_workspace_size(ctypes.byref(d), 512, ctypes.byref(n)) == 0
    for known in (H.HATA_FLAG_TEST_EXPIRE_WAIT, H.HATA_FLAG_ALL_SM_SCAN, 7):
        d.flags = known
        assert H.lib.hata_workspace_size(ctypes.byref(d), 512, ctypes.byref(n)) == 0
    for unknown in (8, 1 | 16, 1 << 30):
        d.flags = unknown
        assert H.lib.hata_workspace_size(ctypes.byref(d), 512, ctypes.byref(n)) == 1
