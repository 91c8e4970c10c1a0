"""Thin Python binding of liblrkv.so (argument marshalling only).

Every entry point mirrors one C function of include/lrkv.h.  PyTorch is used
only to own device memory and to name the current CUDA stream; all
arithmetic of the method runs in the library's kernels.  Importing this
module fails loudly when the compiled library is missing: there is no CPU
fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblrkv.so")

LRKV_BF16, LRKV_F32, LRKV_BF16_Q8, LRKV_BF16_VA = 0, 1, 2, 3
VA_KEEP = 16
HEAD_DIM = 128
PAGE_TOKENS = 64
FULL_RANK_TILE = 32

_STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported configuration",
           -3: "cache capacity exceeded", -4: "workspace too small", -5: "CUDA error"}


class LrkvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {status} ({_STATUS.get(status, 'unknown')})")
        self.status = status


class CacheDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("rank_k", ctypes.c_int32),
                ("rank_v", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("n_sink", ctypes.c_int32), ("window", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
                ("codes", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("anchors", ctypes.c_void_p), ("seq_len", ctypes.c_void_p),
                ("append_counter", ctypes.c_void_p)]


class DenseDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
                ("kv_pages", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("seq_len", ctypes.c_void_p),
                ("append_counter", ctypes.c_void_p)]


EXPORTS = ["lrkv_compress", "lrkv_decode_workspace_bytes", "lrkv_decode_attn",
           "lrkv_oja_update", "lrkv_qr_orthonormalize", "lrkv_dense_append",
           "lrkv_dense_decode_workspace_bytes", "lrkv_dense_decode_attn",
           "lrkv_status_string", "lrkv_version", "lrkv_decode_attn_static",
           "lrkv_rebase_workspace_bytes", "lrkv_rebase", "lrkv_oja_update_chunked",
           "lrkv_compress_amortised", "lrkv_amortise_workspace_bytes", "lrkv_amortise",
           "lrkv_decode_attn_amortised", "lrkv_decode_step"]


def load_library(path: str = _LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with __graft_entry__.build() "
                          "(the latent-KV path has no fallback)")
    lib = ctypes.CDLL(path)
    P, I32, I64, F32, SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                            ctypes.c_float, ctypes.c_size_t)
    sig = {
        "lrkv_compress": (ctypes.c_int, [P, P, P, I32, P, I64, I64, P, P, I64, P]),
        "lrkv_decode_workspace_bytes": (SZ, [P, I32]),
        "lrkv_decode_attn": (ctypes.c_int, [P, P, I32, P, P, I64, F32, P, P, SZ, P]),
        "lrkv_oja_update": (ctypes.c_int, [P, I32, I32, I64, P, I32, I64, I32, F32, I32, I64, P]),
        "lrkv_qr_orthonormalize": (ctypes.c_int, [P, I32, I32, I64, P]),
        "lrkv_oja_update_chunked": (ctypes.c_int,
                                    [P, I32, I32, I64, P, I32, I64, I32, F32, I32, I64, I32, P]),
        "lrkv_dense_append": (ctypes.c_int, [P, P, P, I32, P, I64, I64, P]),
        "lrkv_dense_decode_workspace_bytes": (SZ, [P, I32]),
        "lrkv_dense_decode_attn": (ctypes.c_int, [P, P, I32, F32, P, P, SZ, P]),
        "lrkv_decode_attn_static": (ctypes.c_int, [P, P, I32, P, P, I64, F32, P, P]),
        "lrkv_rebase_workspace_bytes": (SZ, [P]),
        "lrkv_rebase": (ctypes.c_int, [P, P, P, P, P, I64, P, SZ, P]),
        "lrkv_compress_amortised": (ctypes.c_int, [P, P, P, I32, P, I64, I64, P, P, I64, P, P]),
        "lrkv_decode_step": (ctypes.c_int, [P, P, P, I64, I64, P, I32, P, P, I64, F32, P, P, SZ,
                                            P]),
        "lrkv_amortise_workspace_bytes": (SZ, [P]),
        "lrkv_amortise": (ctypes.c_int, [P, P, I32, I64, I64, P, I64, P, P, SZ, P]),
        "lrkv_decode_attn_amortised": (ctypes.c_int,
                                       [P, P, I32, P, P, I64, P, F32, P, P, SZ, P]),
        "lrkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "lrkv_version": (ctypes.c_int, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = load_library()


def _stream(stream=None) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(fn: str, rc: int):
    if rc != 0:
        raise LrkvError(fn, rc)


def _dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return LRKV_BF16
    if dtype == torch.float32:
        return LRKV_F32
    raise ValueError(f"unsupported dtype {dtype}")


def chunk_elems(dtype: torch.dtype) -> int:
    return 16 // torch.empty((), dtype=dtype).element_size()


class LatentCache:
    """Device buffers of one latent cache, laid out as include/lrkv.h says.

    max_tokens bounds the tokens per sequence; the block table maps each
    sequence's latent pages into a shared pool (identity order unless a
    permutation of range(num_pages) is given).
    """

    def __init__(self, B: int, H_kv: int, r_k: int, r_v: int, max_tokens: int,
                 n_sink: int = 0, window: int = 0, dtype=torch.bfloat16,
                 device="cuda", page_perm: Optional[torch.Tensor] = None,
                 int8_codes: bool = False, amortised_values: bool = False):
        ce = chunk_elems(dtype)
        self.B, self.H_kv, self.r_k, self.r_v = B, H_kv, r_k, r_v
        self.n_sink, self.window, self.dtype = n_sink, window, dtype
        self.int8_codes = int8_codes
        max_lat = max(1, max_tokens - n_sink - window)
        self.max_pages = math.ceil(max_lat / PAGE_TOKENS)
        self.num_pages = B * self.max_pages
        self.amortised_values = amortised_values
        if amortised_values:
            # one slab per (page, kv head): key-code chunks, then the value
            # residual slots [r_v / 8][16][8] bf16, slot rows int32 [16] and
            # squared norms fp32 [16]
            assert dtype == torch.bfloat16 and not int8_codes
            self.codes = torch.zeros((self.num_pages, H_kv,
                                      PAGE_TOKENS * r_k * 2 + VA_KEEP * r_v * 2 + VA_KEEP * 8),
                                     dtype=torch.uint8, device=device)
        elif int8_codes:
            # one slab per (page, kv head): int8 code chunks of 16, key codes
            # then value codes, then [64][2] fp32 scales (bf16 inputs)
            assert dtype == torch.bfloat16
            self.codes = torch.zeros((self.num_pages, H_kv, PAGE_TOKENS * (r_k + r_v) + 512),
                                     dtype=torch.uint8, device=device)
        else:
            # one slab per (page, kv head): key-code chunks, then value-code chunks
            self.codes = torch.zeros((self.num_pages, H_kv, (r_k + r_v) // ce, PAGE_TOKENS, ce),
                                     dtype=dtype, device=device)
        ids = torch.arange(self.num_pages, dtype=torch.int32) if page_perm is None else \
            torch.as_tensor(page_perm, dtype=torch.int32)
        self.block_table = ids.reshape(B, self.max_pages).to(device)
        self.anchor_tiles = math.ceil((n_sink + window) / FULL_RANK_TILE)
        na = max(1, self.anchor_tiles)
        self.anchors = torch.zeros((B, H_kv, na, 2 * HEAD_DIM // ce, FULL_RANK_TILE, ce),
                                   dtype=dtype, device=device)
        self.seq_len = torch.zeros(B, dtype=torch.int32, device=device)
        self.append_counter = torch.zeros(B, dtype=torch.int32, device=device)
        code = LRKV_BF16_Q8 if int8_codes else (LRKV_BF16_VA if amortised_values
                                                 else _dtype_code(dtype))
        self.desc = CacheDesc(B, H_kv, HEAD_DIM, r_k, r_v, code, n_sink, window,
                              self.num_pages, self.max_pages, self.codes.data_ptr(),
                              self.block_table.data_ptr(), self.anchors.data_ptr(),
                              self.seq_len.data_ptr(), self.append_counter.data_ptr())

    def nbytes_codes(self) -> int:
        return self.codes.numel() * self.codes.element_size()


def _kv_strides(k: torch.Tensor):
    assert k.dim() == 4 and k.shape[3] == HEAD_DIM and k.stride(3) == 1 and \
        (k.shape[2] <= 1 or k.stride(2) == HEAD_DIM), "k/v must be [B, H_kv, n, 128] rows"
    return k.stride(0), k.stride(1)


def compress(cache: LatentCache, k: torch.Tensor, v: torch.Tensor, P_k: torch.Tensor,
             P_v: torch.Tensor, basis_batch_stride: int = 0, n_new: Optional[torch.Tensor] = None,
             stream=None) -> None:
    """lrkv_compress: append k, v [B, H_kv, n, 128] (n_new[b] <= n tokens of
    sequence b when given) and compress the tokens that become latent."""
    assert k.dtype == cache.dtype and v.dtype == cache.dtype and k.shape == v.shape
    assert P_k.dtype == torch.float32 and P_v.dtype == torch.float32
    ss, hs = _kv_strides(k)
    assert _kv_strides(v) == (ss, hs)
    _check("lrkv_compress", _lib.lrkv_compress(
        ctypes.byref(cache.desc), _ptr(k), _ptr(v), k.shape[2], _ptr(n_new), ss, hs, _ptr(P_k),
        _ptr(P_v),
        basis_batch_stride, _stream(stream)))


def compress_amortised(cache: LatentCache, k: torch.Tensor, v: torch.Tensor,
                       P_k: torch.Tensor, P_v: torch.Tensor, A: torch.Tensor,
                       basis_batch_stride: int = 0, n_new: Optional[torch.Tensor] = None,
                       stream=None) -> None:
    """lrkv_compress_amortised: append to a value-amortised cache whose
    predictors A [B, H_kv, r_k, r_v] exist."""
    assert k.dtype == cache.dtype and v.dtype == cache.dtype and k.shape == v.shape
    assert A.dtype == torch.float32 and A.is_contiguous()
    ss, hs = _kv_strides(k)
    assert _kv_strides(v) == (ss, hs)
    _check("lrkv_compress_amortised", _lib.lrkv_compress_amortised(
        ctypes.byref(cache.desc), _ptr(k), _ptr(v), k.shape[2], _ptr(n_new), ss, hs, _ptr(P_k),
        _ptr(P_v), basis_batch_stride, _ptr(A), _stream(stream)))


def amortise(cache: LatentCache, v: torch.Tensor, P_v: torch.Tensor, A: torch.Tensor,
             basis_batch_stride: int = 0, stream=None) -> None:
    """lrkv_amortise: fit the value predictors A [B, H_kv, r_k, r_v] (fp32,
    written) over the prompt v [B, H_kv, n, 128] and fill the prompt pages'
    residual slots."""
    assert v.dtype == torch.bfloat16 and A.dtype == torch.float32 and A.is_contiguous()
    ss, hs = _kv_strides(v)
    n = int(_lib.lrkv_amortise_workspace_bytes(ctypes.byref(cache.desc)))
    if n == 0:
        raise LrkvError("lrkv_amortise_workspace_bytes", -2)
    ws = torch.zeros(n, dtype=torch.uint8, device=v.device)
    _check("lrkv_amortise", _lib.lrkv_amortise(
        ctypes.byref(cache.desc), _ptr(v), v.shape[2], ss, hs, _ptr(P_v), basis_batch_stride,
        _ptr(A), _ptr(ws), n, _stream(stream)))
    cache._amortise_ws = ws  # kept alive until the stream has used it


def decode_attn_amortised(cache: LatentCache, q: torch.Tensor, P_k: torch.Tensor,
                          P_v: torch.Tensor, A: torch.Tensor, scale: float, o: torch.Tensor,
                          workspace: torch.Tensor, basis_batch_stride: int = 0,
                          stream=None) -> torch.Tensor:
    """lrkv_decode_attn_amortised: o [B, H_q, 128] from q over a
    value-amortised cache with predictors A."""
    assert q.is_contiguous() and o.is_contiguous() and q.dtype == cache.dtype
    _check("lrkv_decode_attn_amortised", _lib.lrkv_decode_attn_amortised(
        ctypes.byref(cache.desc), _ptr(q), q.shape[1], _ptr(P_k), _ptr(P_v), basis_batch_stride,
        _ptr(A), float(scale), _ptr(o), _ptr(workspace), workspace.numel(), _stream(stream)))
    return o


def decode_step(cache: LatentCache, k: torch.Tensor, v: torch.Tensor, q: torch.Tensor,
                P_k: torch.Tensor, P_v: torch.Tensor, scale: float, o: torch.Tensor,
                workspace: torch.Tensor, basis_batch_stride: int = 0,
                stream=None) -> torch.Tensor:
    """lrkv_decode_step: append k, v [B, H_kv, 1, 128] and attend with q
    [B, H_q, 128] -> o."""
    assert k.dtype == cache.dtype and v.dtype == cache.dtype and k.shape == v.shape
    assert k.shape[2] == 1 and q.is_contiguous() and o.is_contiguous() and q.dtype == cache.dtype
    ss, hs = _kv_strides(k)
    assert _kv_strides(v) == (ss, hs)
    _check("lrkv_decode_step", _lib.lrkv_decode_step(
        ctypes.byref(cache.desc), _ptr(k), _ptr(v), ss, hs, _ptr(q), q.shape[1], _ptr(P_k),
        _ptr(P_v), basis_batch_stride, float(scale), _ptr(o), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return o


def decode_workspace_bytes(cache: LatentCache, num_q_heads: int) -> int:
    return int(_lib.lrkv_decode_workspace_bytes(ctypes.byref(cache.desc), num_q_heads))


def decode_workspace(cache: LatentCache, num_q_heads: int, device="cuda") -> torch.Tensor:
    """Zero-filled decode workspace (the library keeps its counters at zero)."""
    n = decode_workspace_bytes(cache, num_q_heads)
    if n == 0:
        raise LrkvError("lrkv_decode_workspace_bytes", -2)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def decode_attn(cache: LatentCache, q: torch.Tensor, P_k: torch.Tensor, P_v: torch.Tensor,
                scale: float, o: torch.Tensor, workspace: torch.Tensor,
                basis_batch_stride: int = 0, stream=None) -> torch.Tensor:
    """lrkv_decode_attn: o [B, H_q, 128] from q [B, H_q, 128]."""
    assert q.is_contiguous() and o.is_contiguous() and q.dtype == cache.dtype
    _check("lrkv_decode_attn", _lib.lrkv_decode_attn(
        ctypes.byref(cache.desc), _ptr(q), q.shape[1], _ptr(P_k), _ptr(P_v), basis_batch_stride,
        float(scale), _ptr(o), _ptr(workspace), workspace.numel(), _stream(stream)))
    return o


def rebase_workspace(cache: LatentCache, device="cuda") -> torch.Tensor:
    """Zero-filled workspace for lrkv_rebase."""
    n = int(_lib.lrkv_rebase_workspace_bytes(ctypes.byref(cache.desc)))
    if n == 0:
        raise LrkvError("lrkv_rebase_workspace_bytes", -2)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def rebase(cache: LatentCache, P_k_old: Optional[torch.Tensor], P_k_new: Optional[torch.Tensor],
           P_v_old: Optional[torch.Tensor], P_v_new: Optional[torch.Tensor],
           workspace: torch.Tensor, basis_batch_stride: int = 0, stream=None) -> None:
    """lrkv_rebase: re-express every stored latent code under the new bases,
    c' = P_new^T (P_old c); a side whose pair is None is left as it is."""
    for t in (P_k_old, P_k_new, P_v_old, P_v_new):
        assert t is None or (t.dtype == torch.float32 and t.is_contiguous())
    _check("lrkv_rebase", _lib.lrkv_rebase(
        ctypes.byref(cache.desc), _ptr(P_k_old), _ptr(P_k_new), _ptr(P_v_old), _ptr(P_v_new),
        basis_batch_stride, _ptr(workspace), workspace.numel(), _stream(stream)))


def decode_attn_static(cache: LatentCache, q: torch.Tensor, P_k: torch.Tensor,
                       P_v: torch.Tensor, scale: float, o: torch.Tensor,
                       basis_batch_stride: int = 0, stream=None) -> torch.Tensor:
    """lrkv_decode_attn_static: decode attention using the library's built-in
    scratch instead of a workspace, for callers that cannot allocate one."""
    assert q.is_contiguous() and o.is_contiguous() and q.dtype == cache.dtype
    _check("lrkv_decode_attn_static", _lib.lrkv_decode_attn_static(
        ctypes.byref(cache.desc), _ptr(q), q.shape[1], _ptr(P_k), _ptr(P_v), basis_batch_stride,
        float(scale), _ptr(o), _stream(stream)))
    return o


def oja_update(P: torch.Tensor, x: torch.Tensor, eta: float, qr_every: int, tokens_seen: int,
               stream=None) -> None:
    """lrkv_oja_update: P [S, 128, r] fp32 in place, x [S, n, 128] rows."""
    assert P.dtype == torch.float32 and P.dim() == 3 and P.shape[1] == HEAD_DIM
    assert P.stride(2) == 1 and P.stride(1) == P.shape[2]
    assert x.dim() == 3 and x.shape[2] == HEAD_DIM and x.stride(2) == 1 and \
        (x.shape[1] <= 1 or x.stride(1) == HEAD_DIM)
    _check("lrkv_oja_update", _lib.lrkv_oja_update(
        _ptr(P), P.shape[0], P.shape[2], P.stride(0), _ptr(x), _dtype_code(x.dtype), x.stride(0),
        x.shape[1], float(eta), int(qr_every), int(tokens_seen), _stream(stream)))


def oja_update_chunked(P: torch.Tensor, x: torch.Tensor, eta: float, qr_every: int,
                       tokens_seen: int, chunk: int = 64, stream=None) -> None:
    """lrkv_oja_update_chunked: the Oja update with P frozen within chunks of
    `chunk` tokens; P [S, 128, r] fp32 in place, x [S, n, 128] rows."""
    assert P.dtype == torch.float32 and P.dim() == 3 and P.shape[1] == HEAD_DIM
    assert P.stride(2) == 1 and P.stride(1) == P.shape[2]
    assert x.dim() == 3 and x.shape[2] == HEAD_DIM and x.stride(2) == 1 and \
        (x.shape[1] <= 1 or x.stride(1) == HEAD_DIM)
    _check("lrkv_oja_update_chunked", _lib.lrkv_oja_update_chunked(
        _ptr(P), P.shape[0], P.shape[2], P.stride(0), _ptr(x), _dtype_code(x.dtype), x.stride(0),
        x.shape[1], float(eta), int(qr_every), int(tokens_seen), int(chunk), _stream(stream)))


def qr_orthonormalize(P: torch.Tensor, stream=None) -> None:
    assert P.dtype == torch.float32 and P.dim() == 3 and P.stride(2) == 1
    _check("lrkv_qr_orthonormalize", _lib.lrkv_qr_orthonormalize(
        _ptr(P), P.shape[0], P.shape[2], P.stride(0), _stream(stream)))


class DenseCache:
    """Full-rank paged bf16/fp32 KV cache of the baseline decode."""

    def __init__(self, B: int, H_kv: int, max_tokens: int, dtype=torch.bfloat16, device="cuda",
                 page_perm: Optional[torch.Tensor] = None):
        ce = chunk_elems(dtype)
        self.B, self.H_kv, self.dtype = B, H_kv, dtype
        self.max_pages = math.ceil(max_tokens / FULL_RANK_TILE)
        self.num_pages = B * self.max_pages
        self.kv_pages = torch.zeros((self.num_pages, H_kv, 2 * HEAD_DIM // ce, FULL_RANK_TILE, ce),
                                    dtype=dtype, device=device)
        ids = torch.arange(self.num_pages, dtype=torch.int32) if page_perm is None else \
            torch.as_tensor(page_perm, dtype=torch.int32)
        self.block_table = ids.reshape(B, self.max_pages).to(device)
        self.seq_len = torch.zeros(B, dtype=torch.int32, device=device)
        self.append_counter = torch.zeros(B, dtype=torch.int32, device=device)
        self.desc = DenseDesc(B, H_kv, HEAD_DIM, _dtype_code(dtype), self.num_pages,
                              self.max_pages, self.kv_pages.data_ptr(),
                              self.block_table.data_ptr(), self.seq_len.data_ptr(),
                              self.append_counter.data_ptr())


def dense_append(cache: DenseCache, k: torch.Tensor, v: torch.Tensor,
                 n_new: Optional[torch.Tensor] = None, stream=None) -> None:
    assert k.dtype == cache.dtype and v.shape == k.shape
    ss, hs = _kv_strides(k)
    assert _kv_strides(v) == (ss, hs)
    _check("lrkv_dense_append", _lib.lrkv_dense_append(
        ctypes.byref(cache.desc), _ptr(k), _ptr(v), k.shape[2], _ptr(n_new), ss, hs,
        _stream(stream)))


def dense_decode_workspace(cache: DenseCache, num_q_heads: int, device="cuda") -> torch.Tensor:
    n = int(_lib.lrkv_dense_decode_workspace_bytes(ctypes.byref(cache.desc), num_q_heads))
    if n == 0:
        raise LrkvError("lrkv_dense_decode_workspace_bytes", -2)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def dense_decode_attn(cache: DenseCache, q: torch.Tensor, scale: float, o: torch.Tensor,
                      workspace: torch.Tensor, stream=None) -> torch.Tensor:
    assert q.is_contiguous() and o.is_contiguous() and q.dtype == cache.dtype
    _check("lrkv_dense_decode_attn", _lib.lrkv_dense_decode_attn(
        ctypes.byref(cache.desc), _ptr(q), q.shape[1], float(scale), _ptr(o), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return o


def workspace_error(workspace: torch.Tensor) -> int:
    """Error word the kernels leave in a decode workspace (0 = ok)."""
    return int(workspace[:4].view(torch.int32).item())


def status_string(status: int) -> str:
    return _lib.lrkv_status_string(status).decode()


def version() -> int:
    return int(_lib.lrkv_version())
