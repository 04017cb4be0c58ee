"""hash_aware_top_b200: Python binding of libhata, the B200 decode-step hot path of
HATA (Hash-Aware Top-k Attention).

The binding only marshals arguments: it checks that every tensor is a
contiguous CUDA tensor of the shape and type the C ABI expects (a wrong pointer
would otherwise be read by a kernel), then passes data pointers and the current
CUDA stream to the library.  All computation happens in the CUDA kernels of
libhata.so; there is no CPU fallback, and importing this package fails loudly
when the library has not been built (python hash_aware_top_b200/build.py).

Function names and argument order follow include/hata.h.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "HataError",
    "Dims",
    "LIB_PATH",
    "lib",
    "dims_for",
    "hata_workspace_size",
    "hata_workspace_init",
    "hata_append_kv",
    "hata_append_kv_paged",
    "hata_prefill_workspace_size",
    "hata_prefill_attention",
    "hata_encode_append",
    "hata_hamming_scores",
    "hata_topk",
    "hata_topk_noalloc",
    "hata_sparse_decode",
    "hata_decode_step",
    "hata_decode_step_qk",
    "hata_decode_step_paged",
    "hata_read_device_status",
    "hata_status_string",
    "hata_version",
    "hata_decode_step_kernel_count",
    "hata_dense_workspace_size",
    "hata_dense_decode",
    "HATA_F32",
    "HATA_BF16",
    "EXPORTED_SYMBOLS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhata.so")

HATA_OK, HATA_ERR_INVALID_ARG, HATA_ERR_UNSUPPORTED, HATA_ERR_CUDA, HATA_ERR_TIMEOUT, HATA_ERR_WORKSPACE = range(6)
HATA_F32, HATA_BF16 = 0, 1
HATA_FLAG_EARLY_PREFETCH = 1
HATA_FLAG_TEST_EXPIRE_WAIT = 2  # test hook: the step's first bounded wait runs out (see include/hata.h)
HATA_FLAG_ALL_SM_SCAN = 4  # the all-SM form of the decode step for any shape it covers

EXPORTED_SYMBOLS = (
    "hata_workspace_size",
    "hata_workspace_init",
    "hata_append_kv",
    "hata_append_kv_paged",
    "hata_prefill_workspace_size",
    "hata_prefill_attention",
    "hata_encode_append",
    "hata_hamming_scores",
    "hata_topk",
    "hata_sparse_decode",
    "hata_decode_step",
    "hata_decode_step_qk",
    "hata_decode_step_paged",
    "hata_read_device_status",
    "hata_status_string",
    "hata_version",
    "hata_decode_step_kernel_count",
    "hata_topk_noalloc",
    "hata_dense_workspace_size",
    "hata_dense_decode",
)


class HataError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {hata_status_string(status)} (status {status})")


class Dims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int),
        ("n_q_heads", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("hash_bits", ctypes.c_int),
        ("max_seq", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("flags", ctypes.c_int),
    ]

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def words(self) -> int:
        return self.hash_bits // 32

    def code_shape(self, *lead) -> tuple:
        """Shape of a code tensor with leading dims `lead`: packed 32-bit words [..., r/32] (int32 or
        uint32), or for r = 16 one 16-bit code per token [...] (int16 or uint16)."""
        return tuple(lead) if self.hash_bits == 16 else tuple(lead) + (self.words,)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == HATA_F32 else torch.bfloat16


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with: python hash_aware_top_b200/build.py")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    DP = ctypes.POINTER(Dims)
    sig = {
        "hata_workspace_size": (I, [DP, I, ctypes.POINTER(S)]),
        "hata_workspace_init": (I, [P, S, P]),
        "hata_append_kv": (I, [DP, P, P, P, P, P, P]),
        "hata_append_kv_paged": (I, [DP, P, P, P, P, P, I, I, P, P]),
        "hata_prefill_workspace_size": (I, [DP, ctypes.POINTER(S)]),
        "hata_prefill_attention": (I, [DP, P, P, P, P, P, P, F, P, P, S, P]),
        "hata_encode_append": (I, [DP, P, I, I, I, P, P, P, I, P, S, P]),
        "hata_hamming_scores": (I, [DP, P, P, P, P, P]),
        "hata_topk": (I, [DP, P, P, I, P, P, P, S, P]),
        "hata_sparse_decode": (I, [DP, P, P, P, P, I, F, P, P, S, P]),
        "hata_decode_step": (I, [DP, P, P, P, P, P, P, I, F, P, P, P, P, S, P]),
        "hata_decode_step_qk": (I, [DP, P, P, P, P, P, P, P, I, F, P, P, P, P, S, P]),
        "hata_decode_step_paged": (I, [DP, P, P, P, P, P, P, P, I, I, P, I, F, P, P, P, P, S, P]),
        "hata_read_device_status": (I, [P, P, ctypes.POINTER(I)]),
        "hata_status_string": (ctypes.c_char_p, [I]),
        "hata_version": (I, []),
        "hata_decode_step_kernel_count": (I, [DP, I]),
        "hata_topk_noalloc": (I, [DP, P, P, I, P, P, P]),
        "hata_dense_workspace_size": (I, [DP, ctypes.POINTER(S)]),
        "hata_dense_decode": (I, [DP, P, P, P, P, F, P, P, S, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


def hata_status_string(status: int) -> str:
    return lib.hata_status_string(int(status)).decode()


def hata_version() -> int:
    return lib.hata_version()


def dims_for(batch, n_q_heads, n_kv_heads, head_dim, hash_bits, max_seq, dtype, flags=0) -> Dims:
    if isinstance(dtype, torch.dtype):
        dtype = HATA_F32 if dtype == torch.float32 else HATA_BF16 if dtype == torch.bfloat16 else -1
    elif isinstance(dtype, str):
        dtype = {"f32": HATA_F32, "bf16": HATA_BF16}[dtype]
    return Dims(batch, n_q_heads, n_kv_heads, head_dim, hash_bits, max_seq, dtype, flags)


def _check(status: int, where: str):
    if status != HATA_OK:
        raise HataError(status, where)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t, name, shape=None, dtype=None, optional=False, numel=None):
    """Device pointer of a contiguous CUDA tensor after shape/type checks (None -> NULL if optional)."""
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} must hold {numel} elements (got {t.numel()})")
    return ctypes.c_void_p(t.data_ptr())


def _codes_dtype(t, dims=None):
    wide = dims is None or dims.hash_bits != 16
    ok = (torch.int32, torch.uint32) if wide else (torch.int16, torch.uint16)
    if t is not None and t.dtype not in ok:
        raise TypeError("codes must be int32 or uint32 tensors holding the packed words"
                        if wide else "16-bit codes must be int16 or uint16 tensors, one code per token")
    return t.dtype if t is not None else None


def hata_workspace_size(dims: Dims, k: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.hata_workspace_size(ctypes.byref(dims), int(k), ctypes.byref(n)), "hata_workspace_size")
    return n.value


def hata_workspace_init(ws: torch.Tensor, stream=None):
    _check(lib.hata_workspace_init(_ptr(ws, "workspace", dtype=torch.uint8), ws.numel(), _stream(stream)),
           "hata_workspace_init")


def hata_append_kv(dims: Dims, new_k, new_v, K, V, seq_lens, stream=None):
    """Write the new token's rows new_k/new_v ([B][Hkv][d]) to slot seq_lens[b] - 1 of K/V."""
    d = dims
    row = (d.batch, d.n_kv_heads, d.head_dim)
    cache = (d.batch, d.n_kv_heads, d.max_seq, d.head_dim)
    _check(
        lib.hata_append_kv(
            ctypes.byref(d),
            _ptr(new_k, "new_k", row, d.torch_dtype), _ptr(new_v, "new_v", row, d.torch_dtype),
            _ptr(K, "K", cache, d.torch_dtype), _ptr(V, "V", cache, d.torch_dtype),
            _ptr(seq_lens, "seq_lens", (d.batch,), torch.int32), _stream(stream)),
        "hata_append_kv")


def hata_append_kv_paged(dims: Dims, new_k, new_v, K_pool, V_pool, block_table, block_size, seq_lens,
                         stream=None):
    """Write the new token's rows new_k/new_v ([B][Hkv][d]) into the paged pools ([n_blocks][Hkv][bs][d])
    at the slot the block table gives for position seq_lens[b] - 1."""
    d = dims
    row = (d.batch, d.n_kv_heads, d.head_dim)
    n_blocks = K_pool.shape[0]
    pool = (n_blocks, d.n_kv_heads, int(block_size), d.head_dim)
    _check(
        lib.hata_append_kv_paged(
            ctypes.byref(d),
            _ptr(new_k, "new_k", row, d.torch_dtype), _ptr(new_v, "new_v", row, d.torch_dtype),
            _ptr(K_pool, "K_pool", pool, d.torch_dtype), _ptr(V_pool, "V_pool", pool, d.torch_dtype),
            _ptr(block_table, "block_table", (d.batch, -(-d.max_seq // int(block_size))), torch.int32),
            int(block_size), int(n_blocks), _ptr(seq_lens, "seq_lens", (d.batch,), torch.int32), _stream(stream)),
        "hata_append_kv_paged")


def hata_prefill_workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.hata_prefill_workspace_size(ctypes.byref(dims), ctypes.byref(n)), "hata_prefill_workspace_size")
    return n.value


def hata_prefill_attention(dims: Dims, q, K, V, W_H, codes, seq_lens, scale, out, ws, stream=None):
    """Causal prefill attention (q/out [B][Hq][max_seq][d], K/V [B][Hkv][max_seq][d], bf16); when codes is
    given (W_H [Hkv][d][r]), every key's code is written as by hata_encode_append."""
    d = dims
    qs = (d.batch, d.n_q_heads, d.max_seq, d.head_dim)
    ks = (d.batch, d.n_kv_heads, d.max_seq, d.head_dim)
    _check(
        lib.hata_prefill_attention(
            ctypes.byref(d), _ptr(q, "q", qs, d.torch_dtype), _ptr(K, "K", ks, d.torch_dtype),
            _ptr(V, "V", ks, d.torch_dtype),
            _ptr(W_H, "W_H", (d.n_kv_heads, d.head_dim, d.hash_bits), torch.float32, optional=codes is None),
            _ptr(codes, "codes", d.code_shape(d.batch, d.n_kv_heads, d.max_seq), _codes_dtype(codes, d),
                 optional=True),
            _ptr(seq_lens, "seq_lens", (d.batch,), torch.int32), float(scale), _ptr(out, "out", qs, d.torch_dtype),
            _ptr(ws, "workspace", dtype=torch.uint8), ws.numel(), _stream(stream)),
        "hata_prefill_attention")


def hata_encode_append(dims: Dims, x, x_heads, x_len, n_tok, seq_end, W_H, codes, codes_len, ws, stream=None):
    """x holds [B][x_heads][x_len][d] elements and codes [B][x_heads][codes_len][r/32] words (any view).

    ws is a uint8 device workspace (at least 16 bytes; a decode-step workspace serves) whose status word
    receives device-side errors; read it with hata_read_device_status."""
    d = dims
    _check(
        lib.hata_encode_append(
            ctypes.byref(d),
            _ptr(x, "x", dtype=d.torch_dtype, numel=d.batch * x_heads * x_len * d.head_dim),
            int(x_heads), int(x_len), int(n_tok),
            _ptr(seq_end, "seq_end", (d.batch,), torch.int32, optional=True),
            _ptr(W_H, "W_H", (d.n_kv_heads, d.head_dim, d.hash_bits), torch.float32),
            _ptr(codes, "codes", dtype=_codes_dtype(codes, d),
                 numel=d.batch * x_heads * codes_len * max(d.words, 1)),
            int(codes_len), _ptr(ws, "workspace", dtype=torch.uint8), ws.numel(), _stream(stream)),
        "hata_encode_append")


def hata_hamming_scores(dims: Dims, qcode, codes, seq_lens, scores, stream=None):
    d = dims
    _check(
        lib.hata_hamming_scores(
            ctypes.byref(d),
            _ptr(qcode, "qcode", d.code_shape(d.batch, d.n_q_heads), _codes_dtype(qcode, d)),
            _ptr(codes, "codes", d.code_shape(d.batch, d.n_kv_heads, d.max_seq), _codes_dtype(codes, d)),
            _ptr(seq_lens, "seq_lens", (d.batch,), torch.int32),
            _ptr(scores, "scores", (d.batch, d.n_kv_heads, d.max_seq), torch.int32),
            _stream(stream)),
        "hata_hamming_scores")


def hata_topk(dims: Dims, scores, seq_lens, k, idx, n_sel, ws, stream=None):
    d = dims
    _check(
        lib.hata_topk(
            ctypes.byref(d),
            _ptr(scores, "scores", (d.batch, d.n_kv_heads, d.max_seq), torch.int32),
            _ptr(seq_lens, "seq_lens", (d.batch,), torch.int32), int(k),
            _ptr(idx, "idx", (d.batch, d.n_kv_heads, k), torch.int32),
            _ptr(n_sel, "n_sel", (d.batch,), torch.int32, optional=True),
            _ptr(ws, "workspace", dtype=torch.uint8), ws.numel(), _stream(stream)),
        "hata_topk")


def hata_topk_noalloc(dims: Dims, scores, seq_lens, k, idx, n_sel, stream=None):
    """hata_topk with the library's built-in scratch instead of a workspace: nothing is allocated.

    For callers that cannot allocate device memory.  Calls on one device share the scratch, so they must not
    overlap on the GPU; the first call on a device should come before any stream capture.
    """
    d = dims
    _check(
        lib.hata_topk_noalloc(
            ctypes.byref(d),
            _ptr(scores, "scores", (d.batch, d.n_kv_heads, d.max_seq), torch.int32),
            _ptr(seq_lens, "seq_lens", (d.batch,), torch.int32), int(k),
            _ptr(idx, "idx", (d.batch, d.n_kv_heads, k), torch.int32),
            _ptr(n_sel, "n_sel", (d.batch,), torch.int32, optional=True), _stream(stream)),
        "hata_topk_noalloc")


def hata_sparse_decode(dims: Dims, q, K, V, idx, k, scale, out, ws, stream=None):
    d = dims
    kv = (d.batch, d.n_kv_heads, d.max_seq, d.head_dim)
    _check(
        lib.hata_sparse_decode(
            ctypes.byref(d),
            _ptr(q, "q", (d.batch, d.n_q_heads, d.head_dim), d.torch_dtype),
            _ptr(K, "K", kv, d.torch_dtype), _ptr(V, "V", kv, d.torch_dtype),
            _ptr(idx, "idx", (d.batch, d.n_kv_heads, k), torch.int32), int(k), float(scale),
            _ptr(out, "out", (d.batch, d.n_q_heads, d.head_dim), d.torch_dtype),
            _ptr(ws, "workspace", dtype=torch.uint8), ws.numel(), _stream(stream)),
        "hata_sparse_decode")


def hata_dense_workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.hata_dense_workspace_size(ctypes.byref(dims), ctypes.byref(n)), "hata_dense_workspace_size")
    return int(n.value)


def hata_dense_decode(dims: Dims, q, K, V, seq_lens, scale, out, ws, stream=None):
    d = dims
    kv = (d.batch, d.n_kv_heads, d.max_seq, d.head_dim)
    _check(
        lib.hata_dense_decode(
            ctypes.byref(d),
            _ptr(q, "q", (d.batch, d.n_q_heads, d.head_dim), d.torch_dtype),
            _ptr(K, "K", kv, d.torch_dtype), _ptr(V, "V", kv, d.torch_dtype),
            _ptr(seq_lens, "seq_lens", (d.batch,), torch.int32, optional=True), float(scale),
            _ptr(out, "out", (d.batch, d.n_q_heads, d.head_dim), d.torch_dtype),
            _ptr(ws, "workspace", dtype=torch.uint8), ws.numel(), _stream(stream)),
        "hata_dense_decode")


def hata_decode_step(dims: Dims, q, K, V, W_H, codes, seq_lens, k, scale, out, qcode_out, idx_out, ws,
                     stream=None):
    d = dims
    kv = (d.batch, d.n_kv_heads, d.max_seq, d.head_dim)
    _check(
        lib.hata_decode_step(
            ctypes.byref(d),
            _ptr(q, "q", (d.batch, d.n_q_heads, d.head_dim), d.torch_dtype),
            _ptr(K, "K", kv, d.torch_dtype), _ptr(V, "V", kv, d.torch_dtype),
            _ptr(W_H, "W_H", (d.n_kv_heads, d.head_dim, d.hash_bits), torch.float32),
            _ptr(codes, "codes", d.code_shape(d.batch, d.n_kv_heads, d.max_seq), _codes_dtype(codes, d)),
            _ptr(seq_lens, "seq_lens", (d.batch,), torch.int32), int(k), float(scale),
            _ptr(out, "out", (d.batch, d.n_q_heads, d.head_dim), d.torch_dtype),
            _ptr(qcode_out, "qcode_out", d.code_shape(d.batch, d.n_q_heads), _codes_dtype(qcode_out, d),
                 optional=True),
            _ptr(idx_out, "idx_out", (d.batch, d.n_kv_heads, k), torch.int32, optional=True),
            _ptr(ws, "workspace", dtype=torch.uint8), ws.numel(), _stream(stream)),
        "hata_decode_step")


def hata_decode_step_qk(dims: Dims, q, K, V, W_q, W_k, codes, seq_lens, k, scale, out, qcode_out, idx_out, ws,
                        stream=None):
    """hata_decode_step with separate query and key encoders (the cache holds codes made with W_k)."""
    d = dims
    kv = (d.batch, d.n_kv_heads, d.max_seq, d.head_dim)
    wshape = (d.n_kv_heads, d.head_dim, d.hash_bits)
    _check(
        lib.hata_decode_step_qk(
            ctypes.byref(d),
            _ptr(q, "q", (d.batch, d.n_q_heads, d.head_dim), d.torch_dtype),
            _ptr(K, "K", kv, d.torch_dtype), _ptr(V, "V", kv, d.torch_dtype),
            _ptr(W_q, "W_q", wshape, torch.float32), _ptr(W_k, "W_k", wshape, torch.float32),
            _ptr(codes, "codes", d.code_shape(d.batch, d.n_kv_heads, d.max_seq), _codes_dtype(codes, d)),
            _ptr(seq_lens, "seq_lens", (d.batch,), torch.int32), int(k), float(scale),
            _ptr(out, "out", (d.batch, d.n_q_heads, d.head_dim), d.torch_dtype),
            _ptr(qcode_out, "qcode_out", d.code_shape(d.batch, d.n_q_heads), _codes_dtype(qcode_out, d),
                 optional=True),
            _ptr(idx_out, "idx_out", (d.batch, d.n_kv_heads, k), torch.int32, optional=True),
            _ptr(ws, "workspace", dtype=torch.uint8), ws.numel(), _stream(stream)),
        "hata_decode_step_qk")


def hata_decode_step_paged(dims: Dims, q, K_pool, V_pool, W_q, W_k, codes_pool, block_table, block_size, seq_lens, k,
                           scale, out, qcode_out, idx_out, ws, stream=None):
    """The decode step over a paged cache: pools [n_blocks][Hkv][block_size][...], block_table [B][max_blocks]."""
    d = dims
    n_blocks = int(K_pool.shape[0]) if K_pool is not None else 0
    bs = int(block_size)
    pool = (n_blocks, d.n_kv_heads, bs, d.head_dim)
    wshape = (d.n_kv_heads, d.head_dim, d.hash_bits)
    max_blocks = (d.max_seq + bs - 1) // bs if bs > 0 else 0
    _check(
        lib.hata_decode_step_paged(
            ctypes.byref(d),
            _ptr(q, "q", (d.batch, d.n_q_heads, d.head_dim), d.torch_dtype),
            _ptr(K_pool, "K_pool", pool, d.torch_dtype), _ptr(V_pool, "V_pool", pool, d.torch_dtype),
            _ptr(W_q, "W_q", wshape, torch.float32), _ptr(W_k, "W_k", wshape, torch.float32),
            _ptr(codes_pool, "codes_pool", d.code_shape(n_blocks, d.n_kv_heads, bs), _codes_dtype(codes_pool, d)),
            _ptr(block_table, "block_table", (d.batch, max_blocks), torch.int32), bs, n_blocks,
            _ptr(seq_lens, "seq_lens", (d.batch,), torch.int32), int(k), float(scale),
            _ptr(out, "out", (d.batch, d.n_q_heads, d.head_dim), d.torch_dtype),
            _ptr(qcode_out, "qcode_out", d.code_shape(d.batch, d.n_q_heads), _codes_dtype(qcode_out, d),
                 optional=True),
            _ptr(idx_out, "idx_out", (d.batch, d.n_kv_heads, k), torch.int32, optional=True),
            _ptr(ws, "workspace", dtype=torch.uint8), ws.numel(), _stream(stream)),
        "hata_decode_step_paged")


def hata_read_device_status(ws, stream=None) -> int:
    v = ctypes.c_int(0)
    _check(lib.hata_read_device_status(_ptr(ws, "workspace", dtype=torch.uint8), _stream(stream), ctypes.byref(v)),
           "hata_read_device_status")
    return v.value


def hata_decode_step_kernel_count(dims: Dims, k: int) -> int:
    n = lib.hata_decode_step_kernel_count(ctypes.byref(dims), int(k))
    if n < 0:
        raise HataError(HATA_ERR_INVALID_ARG, "hata_decode_step_kernel_count")
    return n


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
