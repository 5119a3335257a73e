"""Thin Python binding of ``libnosa_b200.so`` (the C ABI in ``include/nosa.h``).

Argument marshalling only: every function takes torch tensors, checks device,
dtype and contiguity, passes raw pointers and the current CUDA stream to the
C entry point of the same name, and raises :class:`NosaError` on a non-zero
status.  All arithmetic runs in the library's CUDA kernels; there is no CPU
path, and importing the library fails loudly when it has not been built.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnosa_b200.so")

NOSA_OK = 0
NOSA_ERR_INVALID_ARG = 1
NOSA_ERR_UNSUPPORTED = 2
NOSA_ERR_WORKSPACE = 3
NOSA_ERR_CUDA = 4
NOSA_ERR_DEVICE_CHECK = 5
NOSA_ERR_TIMEOUT = 6

NOSA_DEV_BAD_LENGTH = 0x1
NOSA_DEV_NC_CAP = 0x2
NOSA_DEV_BAD_INDEX = 0x4
NOSA_DEV_BAD_COUNT = 0x8
NOSA_DEV_MAX_NEW_KEYS = 0x10
NOSA_DEV_APPEND_ONE = 0x20
NOSA_DEV_MAX_LEN = 0x40
NOSA_DEV_CACHE_ROWS = 0x80
NOSA_DEV_TIMEOUT = 0x80000000


class NosaError(RuntimeError):
    def __init__(self, code: int, func: str, detail: str):
        self.code = code
        super().__init__(f"{func}: {_status_string(code)} (code {code}): {detail}")


class nosa_params(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("pool_kernel", ctypes.c_int),
                ("pool_stride", ctypes.c_int), ("block_size", ctypes.c_int),
                ("local_blocks", ctypes.c_int), ("topk", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("pooled_bf16", ctypes.c_int),
                ("kv_int8", ctypes.c_int)]

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def pooled_dtype(self):
        """torch dtype of the pooled keys: float32, or bfloat16 when pooled_bf16."""
        return torch.bfloat16 if self.pooled_bf16 else torch.float32


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_I64 = ctypes.c_int64

_SIGNATURES = {
    "nosa_default_params": (None, [_P]),
    "nosa_kv_int8_bytes": (_SZ, [_I64, _I]),
    "nosa_prefill_workspace_size": (_SZ, [_P, _I, _I]),
    "nosa_sparse_prefill": (_I, [_P, _P, _P, _P, _I64, _P, _P, _P, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "nosa_sparse_prefill_paged": (_I, [_P, _P, _P, _P, _I64, _P, _I, _P, _P, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P,
                                       _SZ, _P]),
    "nosa_quantize_kv_int8": (_I, [_P, _P, _P, _I64, _I64, _I64, _P]),
    "nosa_workspace_size": (_SZ, [_P, _I, _I]),
    "nosa_workspace_init": (_I, [_P, _SZ, _P]),
    "nosa_pool_append": (_I, [_P, _P, _P, _I64, _P, _P, _P, _I, _P, _I, _I, _P, _P, _P, _SZ, _P]),
    "nosa_block_select": (_I, [_P, _P, _P, _I, _P, _I, _I, _P, _I, _P, _P, _I, _P, _P, _P, _SZ, _P]),
    "nosa_sparse_decode": (_I, [_P, _P, _P, _P, _I64, _P, _P, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "nosa_decode_step_device": (_I, [_P, _P, _P, _P, _P, _P, _I64, _P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "nosa_decode_step_device_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I64, _P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _P]),
    "nosa_pool_append_paged": (_I, [_P, _P, _P, _I64, _P, _I, _P, _P, _I, _P, _I, _I, _P, _P, _P, _SZ, _P]),
    "nosa_sparse_decode_paged": (_I, [_P, _P, _P, _P, _I64, _P, _I, _P, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "nosa_decode_step_device_paged": (_I, [_P, _P, _P, _P, _P, _P, _I64, _P, _I, _P, _I, _I, _P, _I, _P, _P, _P,
                                           _P, _P, _SZ, _P]),
    "nosa_decode_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _I64, _P, _P, _I, _I, _P, _I, _P, _P, _P, _SZ, _P]),
    "nosa_decode_step_packed": (_I, [_P, _P, _P, _P, _P, _I64, _P, _P, _I, _I, _P, _I, _P, _P, _P, _SZ, _P]),
    "nosa_read_device_status": (_I, [_P, _SZ, _P]),
    "nosa_last_device_bits": (ctypes.c_uint32, []),
    "nosa_selftest_wait_timeout": (_I, [_P, _SZ, ctypes.c_uint32, _P]),
    "nosa_status_string": (ctypes.c_char_p, [_I]),
    "nosa_last_error": (ctypes.c_char_p, []),
}


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m long_context_decode_nosa_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _status_string(code: int) -> str:
    try:
        return lib().nosa_status_string(code).decode()
    except Exception:  # noqa: BLE001 -- message formatting only
        return "status"


def _check(rc: int, func: str):
    if rc != NOSA_OK:
        raise NosaError(rc, func, lib().nosa_last_error().decode())


def params(num_q_heads: int = 16, num_kv_heads: int = 2, *, topk: int = 64,
           local_blocks: int = 16, softmax_scale: float = 0.0, head_dim: int = 128,
           pool_kernel: int = 32, pool_stride: int = 16, block_size: int = 64,
           pooled_bf16: bool = False, kv_int8: bool = False) -> nosa_params:
    return nosa_params(num_q_heads, num_kv_heads, head_dim, pool_kernel, pool_stride, block_size,
                       local_blocks, topk, softmax_scale, int(pooled_bf16), int(kv_int8))


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor", cuda=True):
    if t is None:
        return None
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not cuda and t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class Int8KvCache:
    """An INT8 K or V cache (params kv_int8) in the buffer layout of nosa.h:
    int8 codes [rows, Hkv, 128], then fp32 scales [Hkv, scale_stride]
    (scale_stride = rows rounded up to 4).  Row r of head h holds the values
    scales[h, r] * codes[r, h, :].  Pass it wherever a call takes k_cache or
    v_cache."""

    def __init__(self, rows: int, num_kv_heads: int, device="cuda"):
        n = lib().nosa_kv_int8_bytes(rows, num_kv_heads)
        if n == 0:
            raise NosaError(NOSA_ERR_INVALID_ARG, "nosa_kv_int8_bytes", "invalid rows / heads")
        self.rows, self.num_kv_heads = rows, num_kv_heads
        self.scale_stride = (rows + 3) // 4 * 4
        self.buffer = torch.zeros(n, dtype=torch.uint8, device=device)

    @property
    def shape(self):
        return (self.rows, self.num_kv_heads, 128)

    @property
    def is_cuda(self) -> bool:
        return self.buffer.is_cuda

    @property
    def codes(self) -> torch.Tensor:
        n = self.rows * self.num_kv_heads * 128
        return self.buffer[:n].view(torch.int8).view(self.rows, self.num_kv_heads, 128)

    @property
    def scales(self) -> torch.Tensor:
        off = self.rows * self.num_kv_heads * 128
        n = self.num_kv_heads * self.scale_stride * 4
        return self.buffer[off:off + n].view(torch.float32).view(self.num_kv_heads, self.scale_stride)

    def row_scales(self) -> torch.Tensor:
        """Scales as [rows, Hkv] (the token-major view)."""
        return self.scales[:, :self.rows].t()

    def clone(self) -> "Int8KvCache":
        c = Int8KvCache.__new__(Int8KvCache)
        c.rows, c.num_kv_heads, c.scale_stride = self.rows, self.num_kv_heads, self.scale_stride
        c.buffer = self.buffer.clone()
        return c

    @classmethod
    def from_bf16(cls, p: nosa_params, cache: torch.Tensor, stream=None) -> "Int8KvCache":
        """Quantizes a whole bf16 cache [rows, Hkv, 128] on the GPU."""
        c = cls(cache.shape[0], cache.shape[1], device=cache.device)
        nosa_quantize_kv_int8(p, cache, c, stream=stream)
        return c


def nosa_quantize_kv_int8(p: nosa_params, src: torch.Tensor, cache: Int8KvCache, *, row0: int = 0, stream=None):
    """Quantizes bf16 rows src [n, Hkv, 128] into rows row0 .. row0 + n - 1."""
    if src.shape[1:] != (cache.num_kv_heads, 128):
        raise ValueError("src must be [n, Hkv, 128] with the cache's Hkv")
    rc = lib().nosa_quantize_kv_int8(ctypes.byref(p), _ptr(src, torch.bfloat16, "src"),
                                     _ptr(cache.buffer, torch.uint8, "cache"), cache.rows, row0, src.shape[0],
                                     _stream(stream))
    _check(rc, "nosa_quantize_kv_int8")


def _cache(p: nosa_params, c, name: str):
    """Pointer of a K/V cache argument: a bf16 tensor, or an Int8KvCache when
    params.kv_int8."""
    if c is None:
        return None
    if p.kv_int8:
        if not isinstance(c, Int8KvCache):
            raise TypeError(f"{name} must be an Int8KvCache when params.kv_int8 is set")
        return _ptr(c.buffer, torch.uint8, name)
    if isinstance(c, Int8KvCache):
        raise TypeError(f"{name} is an Int8KvCache but params.kv_int8 is not set")
    return _ptr(c, torch.bfloat16, name)


def n_windows(L: int) -> int:
    return (L - 32) // 16 + 1 if L >= 32 else 0


def n_blocks(L: int) -> int:
    return (L + 63) // 64


def workspace_size(p: nosa_params, batch: int, max_seq_len: int) -> int:
    n = lib().nosa_workspace_size(ctypes.byref(p), batch, max_seq_len)
    if n == 0:
        raise NosaError(NOSA_ERR_INVALID_ARG, "nosa_workspace_size", "invalid parameters")
    return n


def nosa_workspace_init(ws: torch.Tensor, stream=None):
    _check(lib().nosa_workspace_init(_ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)),
           "nosa_workspace_init")


def workspace(p: nosa_params, batch: int, max_seq_len: int, device="cuda", stream=None) -> torch.Tensor:
    """A zero-initialised workspace tensor (uint8) for these shapes."""
    n = workspace_size(p, batch, max_seq_len)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    nosa_workspace_init(ws, stream)
    return ws


def nosa_pool_append(p: nosa_params, k_cache: torch.Tensor, v_cache: Optional[torch.Tensor],
                     seq_start: torch.Tensor, len_new: torch.Tensor, pooled: torch.Tensor, *,
                     len_old: Optional[torch.Tensor] = None, max_new_keys: int = 1,
                     k_new: Optional[torch.Tensor] = None, v_new: Optional[torch.Tensor] = None,
                     ws: Optional[torch.Tensor] = None, stream=None):
    batch = len_new.shape[0]
    rc = lib().nosa_pool_append(
        ctypes.byref(p), _cache(p, k_cache, "k_cache"), _cache(p, v_cache, "v_cache"),
        k_cache.shape[0], _ptr(seq_start, torch.int64, "seq_start"), _ptr(len_old, torch.int32, "len_old"),
        _ptr(len_new, torch.int32, "len_new"), batch, _ptr(pooled, p.pooled_dtype, "pooled"),
        pooled.shape[2], max_new_keys, _ptr(k_new, torch.bfloat16, "k_new"),
        _ptr(v_new, torch.bfloat16, "v_new"), _ptr(ws, torch.uint8, "ws"),
        0 if ws is None else ws.numel(), _stream(stream))
    _check(rc, "nosa_pool_append")


def nosa_block_select(p: nosa_params, q: Optional[torch.Tensor], pooled: Optional[torch.Tensor],
                      seq_len: torch.Tensor, max_seq_len: int, sel_idx: torch.Tensor,
                      sel_cnt: torch.Tensor, ws: torch.Tensor, *,
                      block_scores_in: Optional[torch.Tensor] = None,
                      comp_scores_out: Optional[torch.Tensor] = None,
                      block_scores_out: Optional[torch.Tensor] = None, stream=None):
    batch = seq_len.shape[0]
    nc_cap = pooled.shape[2] if pooled is not None else (comp_scores_out.shape[2] if comp_scores_out is not None else 0)
    rc = lib().nosa_block_select(
        ctypes.byref(p), _ptr(q, torch.bfloat16, "q"), _ptr(pooled, p.pooled_dtype, "pooled"), nc_cap,
        _ptr(seq_len, torch.int32, "seq_len"), batch, max_seq_len,
        _ptr(block_scores_in, torch.float32, "block_scores_in"),
        0 if block_scores_in is None else block_scores_in.shape[2],
        _ptr(comp_scores_out, torch.float32, "comp_scores_out"),
        _ptr(block_scores_out, torch.float32, "block_scores_out"),
        0 if block_scores_out is None else block_scores_out.shape[2],
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(rc, "nosa_block_select")


def nosa_sparse_decode(p: nosa_params, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                       seq_start: torch.Tensor, seq_len: torch.Tensor, max_seq_len: int,
                       sel_idx: torch.Tensor, sel_cnt: torch.Tensor, out: torch.Tensor,
                       ws: torch.Tensor, *, lse: Optional[torch.Tensor] = None, stream=None):
    if sel_idx.shape[-1] != p.topk:
        raise ValueError("sel_idx's last dimension must equal params.topk")
    batch = seq_len.shape[0]
    rc = lib().nosa_sparse_decode(
        ctypes.byref(p), _ptr(q, torch.bfloat16, "q"), _cache(p, k_cache, "k_cache"),
        _cache(p, v_cache, "v_cache"), k_cache.shape[0], _ptr(seq_start, torch.int64, "seq_start"),
        _ptr(seq_len, torch.int32, "seq_len"), batch, max_seq_len,
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"),
        _ptr(out, torch.bfloat16, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(rc, "nosa_sparse_decode")


def nosa_decode_step_device(p: nosa_params, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                            seq_start: torch.Tensor, seq_len: torch.Tensor, max_seq_len: int,
                            pooled: torch.Tensor, sel_idx: torch.Tensor, sel_cnt: torch.Tensor,
                            out: torch.Tensor, ws: torch.Tensor, *, k_new: Optional[torch.Tensor] = None,
                            v_new: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                            stream=None):
    """Whole decode step on device buffers in one fused launch."""
    if sel_idx.shape[-1] != p.topk:
        raise ValueError("sel_idx's last dimension must equal params.topk")
    batch = seq_len.shape[0]
    rc = lib().nosa_decode_step_device(
        ctypes.byref(p), _ptr(q, torch.bfloat16, "q"), _ptr(k_new, torch.bfloat16, "k_new"),
        _ptr(v_new, torch.bfloat16, "v_new"), _cache(p, k_cache, "k_cache"),
        _cache(p, v_cache, "v_cache"), k_cache.shape[0], _ptr(seq_start, torch.int64, "seq_start"),
        _ptr(seq_len, torch.int32, "seq_len"), batch, max_seq_len, _ptr(pooled, p.pooled_dtype, "pooled"),
        pooled.shape[2], _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"),
        _ptr(out, torch.bfloat16, "out"), _ptr(lse, torch.float32, "lse"), _ptr(ws, torch.uint8, "ws"),
        ws.numel(), _stream(stream))
    _check(rc, "nosa_decode_step_device")


# ----------------------------------------------------------------------------- sparse prefill

def prefill_workspace(p: nosa_params, total_q: int, max_seq_len: int, device="cuda", stream=None) -> torch.Tensor:
    """A zero-initialised workspace for nosa_sparse_prefill over total_q query rows."""
    n = lib().nosa_prefill_workspace_size(ctypes.byref(p), total_q, max_seq_len)
    if n == 0:
        raise NosaError(NOSA_ERR_INVALID_ARG, "nosa_prefill_workspace_size", "invalid parameters")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    nosa_workspace_init(ws, stream)
    return ws


def nosa_sparse_prefill(p: nosa_params, q: torch.Tensor, k_cache, v_cache, seq_start: torch.Tensor,
                        q_start: torch.Tensor, q_pos: torch.Tensor, max_seq_len: int, pooled: torch.Tensor,
                        sel_idx: torch.Tensor, sel_cnt: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, *,
                        lse: Optional[torch.Tensor] = None, stream=None):
    """Sparse prefill: every row of q (sequence s owns rows q_start[s] ..
    q_start[s+1]-1 at positions q_pos[s] + r) is a decode query of its own
    prefix (L = position + 1) against sequence s's cache and pooled keys."""
    if sel_idx.shape[-1] != p.topk:
        raise ValueError("sel_idx's last dimension must equal params.topk")
    batch = q_pos.shape[0]
    if q_start.shape[0] != batch + 1:
        raise ValueError("q_start must have batch + 1 entries")
    rc = lib().nosa_sparse_prefill(
        ctypes.byref(p), _ptr(q, torch.bfloat16, "q"), _cache(p, k_cache, "k_cache"), _cache(p, v_cache, "v_cache"),
        k_cache.shape[0], _ptr(seq_start, torch.int64, "seq_start"), _ptr(q_start, torch.int32, "q_start"),
        _ptr(q_pos, torch.int32, "q_pos"), batch, q.shape[0], max_seq_len, _ptr(pooled, p.pooled_dtype, "pooled"),
        pooled.shape[2], _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"),
        _ptr(out, torch.bfloat16, "out"), _ptr(lse, torch.float32, "lse"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream(stream))
    _check(rc, "nosa_sparse_prefill")


def nosa_sparse_prefill_paged(p: nosa_params, q: torch.Tensor, k_cache, v_cache, page_table: torch.Tensor,
                              q_start: torch.Tensor, q_pos: torch.Tensor, max_seq_len: int, pooled: torch.Tensor,
                              sel_idx: torch.Tensor, sel_cnt: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, *,
                              lse: Optional[torch.Tensor] = None, stream=None):
    """nosa_sparse_prefill over a paged cache (page_table int32 [batch, max_pages])."""
    if sel_idx.shape[-1] != p.topk:
        raise ValueError("sel_idx's last dimension must equal params.topk")
    batch = q_pos.shape[0]
    if q_start.shape[0] != batch + 1 or page_table.shape[0] != batch:
        raise ValueError("q_start must have batch + 1 entries and page_table batch rows")
    rc = lib().nosa_sparse_prefill_paged(
        ctypes.byref(p), _ptr(q, torch.bfloat16, "q"), _cache(p, k_cache, "k_cache"), _cache(p, v_cache, "v_cache"),
        _pages(k_cache), _ptr(page_table, torch.int32, "page_table"), page_table.shape[1],
        _ptr(q_start, torch.int32, "q_start"), _ptr(q_pos, torch.int32, "q_pos"), batch, q.shape[0], max_seq_len,
        _ptr(pooled, p.pooled_dtype, "pooled"), pooled.shape[2], _ptr(sel_idx, torch.int32, "sel_idx"),
        _ptr(sel_cnt, torch.int32, "sel_cnt"), _ptr(out, torch.bfloat16, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(rc, "nosa_sparse_prefill_paged")


# ----------------------------------------------------------------------------- paged KV cache
# Caches as pools of 64-token pages ([num_pages * 64, Hkv, 128]); page_table
# int32 [batch, max_pages]: token t of sequence i in row
# page_table[i, t // 64] * 64 + t % 64.

def _pages(k_cache: torch.Tensor) -> int:
    if k_cache.shape[0] % 64:
        raise ValueError("a paged cache holds whole 64-token pages")
    return k_cache.shape[0] // 64


def nosa_pool_append_paged(p: nosa_params, k_cache: torch.Tensor, v_cache: Optional[torch.Tensor],
                           page_table: torch.Tensor, len_new: torch.Tensor, pooled: torch.Tensor, *,
                           len_old: Optional[torch.Tensor] = None, max_new_keys: int = 1,
                           k_new: Optional[torch.Tensor] = None, v_new: Optional[torch.Tensor] = None,
                           ws: Optional[torch.Tensor] = None, stream=None):
    batch = len_new.shape[0]
    rc = lib().nosa_pool_append_paged(
        ctypes.byref(p), _cache(p, k_cache, "k_cache"), _cache(p, v_cache, "v_cache"),
        _pages(k_cache), _ptr(page_table, torch.int32, "page_table"), page_table.shape[1],
        _ptr(len_old, torch.int32, "len_old"), _ptr(len_new, torch.int32, "len_new"), batch,
        _ptr(pooled, p.pooled_dtype, "pooled"), pooled.shape[2], max_new_keys,
        _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
        _ptr(ws, torch.uint8, "ws"), ws.numel() if ws is not None else 0, _stream(stream))
    _check(rc, "nosa_pool_append_paged")


def nosa_sparse_decode_paged(p: nosa_params, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                             page_table: torch.Tensor, seq_len: torch.Tensor, max_seq_len: int,
                             sel_idx: torch.Tensor, sel_cnt: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, *,
                             lse: Optional[torch.Tensor] = None, stream=None):
    if sel_idx.shape[-1] != p.topk:
        raise ValueError("sel_idx's last dimension must equal params.topk")
    batch = seq_len.shape[0]
    rc = lib().nosa_sparse_decode_paged(
        ctypes.byref(p), _ptr(q, torch.bfloat16, "q"), _cache(p, k_cache, "k_cache"),
        _cache(p, v_cache, "v_cache"), _pages(k_cache), _ptr(page_table, torch.int32, "page_table"),
        page_table.shape[1], _ptr(seq_len, torch.int32, "seq_len"), batch, max_seq_len,
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"),
        _ptr(out, torch.bfloat16, "out"), _ptr(lse, torch.float32, "lse"), _ptr(ws, torch.uint8, "ws"),
        ws.numel(), _stream(stream))
    _check(rc, "nosa_sparse_decode_paged")


def nosa_decode_step_device_paged(p: nosa_params, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                  page_table: torch.Tensor, seq_len: torch.Tensor, max_seq_len: int,
                                  pooled: torch.Tensor, sel_idx: torch.Tensor, sel_cnt: torch.Tensor,
                                  out: torch.Tensor, ws: torch.Tensor, *, k_new: Optional[torch.Tensor] = None,
                                  v_new: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                                  stream=None):
    if sel_idx.shape[-1] != p.topk:
        raise ValueError("sel_idx's last dimension must equal params.topk")
    batch = seq_len.shape[0]
    rc = lib().nosa_decode_step_device_paged(
        ctypes.byref(p), _ptr(q, torch.bfloat16, "q"), _ptr(k_new, torch.bfloat16, "k_new"),
        _ptr(v_new, torch.bfloat16, "v_new"), _cache(p, k_cache, "k_cache"),
        _cache(p, v_cache, "v_cache"), _pages(k_cache), _ptr(page_table, torch.int32, "page_table"),
        page_table.shape[1], _ptr(seq_len, torch.int32, "seq_len"), batch, max_seq_len,
        _ptr(pooled, p.pooled_dtype, "pooled"), pooled.shape[2], _ptr(sel_idx, torch.int32, "sel_idx"),
        _ptr(sel_cnt, torch.int32, "sel_cnt"), _ptr(out, torch.bfloat16, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(rc, "nosa_decode_step_device_paged")


def nosa_decode_step_device_noalloc(p: nosa_params, q: torch.Tensor, k_cache: torch.Tensor,
                                    v_cache: torch.Tensor, seq_start: torch.Tensor, seq_len: torch.Tensor,
                                    max_seq_len: int, pooled: torch.Tensor, sel_idx: torch.Tensor,
                                    sel_cnt: torch.Tensor, out: torch.Tensor, *,
                                    k_new: Optional[torch.Tensor] = None, v_new: Optional[torch.Tensor] = None,
                                    lse: Optional[torch.Tensor] = None, stream=None):
    """The fused decode step without a workspace: its scratch is the library's
    own fixed device array (for callers that cannot allocate device memory)."""
    if sel_idx.shape[-1] != p.topk:
        raise ValueError("sel_idx's last dimension must equal params.topk")
    batch = seq_len.shape[0]
    rc = lib().nosa_decode_step_device_noalloc(
        ctypes.byref(p), _ptr(q, torch.bfloat16, "q"), _ptr(k_new, torch.bfloat16, "k_new"),
        _ptr(v_new, torch.bfloat16, "v_new"), _cache(p, k_cache, "k_cache"),
        _cache(p, v_cache, "v_cache"), k_cache.shape[0], _ptr(seq_start, torch.int64, "seq_start"),
        _ptr(seq_len, torch.int32, "seq_len"), batch, max_seq_len, _ptr(pooled, p.pooled_dtype, "pooled"),
        pooled.shape[2], _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"),
        _ptr(out, torch.bfloat16, "out"), _ptr(lse, torch.float32, "lse"), _stream(stream))
    _check(rc, "nosa_decode_step_device_noalloc")


def nosa_decode_step(p: nosa_params, q_host: torch.Tensor, k_new_host: torch.Tensor,
                     v_new_host: torch.Tensor, out_host: torch.Tensor, k_cache: torch.Tensor,
                     v_cache: torch.Tensor, seq_start: torch.Tensor, seq_len: torch.Tensor,
                     max_seq_len: int, pooled: torch.Tensor, sel_idx: torch.Tensor,
                     sel_cnt: torch.Tensor, ws: torch.Tensor, stream=None):
    """Whole decode step from host buffers (pinned for asynchronous copies);
    out_host is valid once the stream has synchronised."""
    batch = seq_len.shape[0]
    rc = lib().nosa_decode_step(
        ctypes.byref(p), _ptr(q_host, torch.bfloat16, "q_host", cuda=False),
        _ptr(k_new_host, torch.bfloat16, "k_new_host", cuda=False),
        _ptr(v_new_host, torch.bfloat16, "v_new_host", cuda=False),
        _ptr(out_host, torch.bfloat16, "out_host", cuda=False),
        _cache(p, k_cache, "k_cache"), _cache(p, v_cache, "v_cache"),
        k_cache.shape[0], _ptr(seq_start, torch.int64, "seq_start"), _ptr(seq_len, torch.int32, "seq_len"),
        batch, max_seq_len, _ptr(pooled, p.pooled_dtype, "pooled"), pooled.shape[2],
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(rc, "nosa_decode_step")


def nosa_decode_step_packed(p: nosa_params, qkv_host: torch.Tensor, out_host: torch.Tensor, k_cache: torch.Tensor,
                            v_cache: torch.Tensor, seq_start: torch.Tensor, seq_len: torch.Tensor, max_seq_len: int,
                            pooled: torch.Tensor, sel_idx: torch.Tensor, sel_cnt: torch.Tensor, ws: torch.Tensor,
                            stream=None):
    """nosa_decode_step with q, k_new and v_new back to back in one host
    buffer (bf16, batch * (Hq + 2 Hkv) * 128 elements), copied in once."""
    batch = seq_len.shape[0]
    need = batch * (p.num_q_heads + 2 * p.num_kv_heads) * 128
    if not qkv_host.is_contiguous() or qkv_host.numel() != need:
        raise ValueError(f"qkv_host must be a contiguous buffer of {need} bf16 values")
    rc = lib().nosa_decode_step_packed(
        ctypes.byref(p), _ptr(qkv_host, torch.bfloat16, "qkv_host", cuda=False),
        _ptr(out_host, torch.bfloat16, "out_host", cuda=False),
        _cache(p, k_cache, "k_cache"), _cache(p, v_cache, "v_cache"),
        k_cache.shape[0], _ptr(seq_start, torch.int64, "seq_start"), _ptr(seq_len, torch.int32, "seq_len"),
        batch, max_seq_len, _ptr(pooled, p.pooled_dtype, "pooled"), pooled.shape[2],
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(rc, "nosa_decode_step_packed")


def nosa_read_device_status(ws: torch.Tensor, stream=None):
    """(status code, raw device bits); synchronises the stream and clears the word."""
    rc = lib().nosa_read_device_status(_ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    return rc, int(lib().nosa_last_device_bits())


def nosa_selftest_wait_timeout(ws: torch.Tensor, max_iters: int = 1000, stream=None):
    _check(lib().nosa_selftest_wait_timeout(_ptr(ws, torch.uint8, "ws"), ws.numel(), max_iters,
                                            _stream(stream)), "nosa_selftest_wait_timeout")


class DecodeState:
    """Device buffers for repeated decode steps of one layer: pooled keys,
    selection, output and workspace, sized for ``batch`` sequences of at most
    ``max_seq_len`` tokens.  A convenience over the C entry points."""

    def __init__(self, p: nosa_params, batch: int, max_seq_len: int, device="cuda"):
        self.p = p
        self.batch = batch
        self.max_seq_len = max_seq_len
        self.nc_cap = max(1, n_windows(max_seq_len))
        self.pooled = torch.zeros(batch, p.num_kv_heads, self.nc_cap, 128, dtype=p.pooled_dtype, device=device)
        self.sel_idx = torch.full((batch, p.num_kv_heads, p.topk), -1, dtype=torch.int32, device=device)
        self.sel_cnt = torch.zeros(batch, p.num_kv_heads, dtype=torch.int32, device=device)
        self.out = torch.empty(batch, p.num_q_heads, 128, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(batch, p.num_q_heads, dtype=torch.float32, device=device)
        self.ws = workspace(p, batch, max_seq_len, device)

    def rebuild_pooled(self, k_cache, seq_start, seq_len, stream=None):
        """Pool every complete window of [0, seq_len) (the resume path)."""
        nosa_pool_append(self.p, k_cache, None, seq_start, seq_len, self.pooled,
                         len_old=torch.zeros_like(seq_len), max_new_keys=self.nc_cap, ws=self.ws,
                         stream=stream)

    def step(self, q, k_cache, v_cache, seq_start, seq_len, *, append=True, stream=None,
             with_lse=False, fused=False, k_new=None, v_new=None):
        """One decode step on device-resident inputs: (when ``append``) write the
        new token's K/V rows if given and pool the window the newest token
        completes, then select and attend.  ``fused`` runs it as one launch.
        Returns ``out``."""
        lse = self.lse if with_lse else None
        if fused:
            if not append:
                raise ValueError("the fused step always pools the newest token's window")
            nosa_decode_step_device(self.p, q, k_cache, v_cache, seq_start, seq_len, self.max_seq_len,
                                    self.pooled, self.sel_idx, self.sel_cnt, self.out, self.ws,
                                    k_new=k_new, v_new=v_new, lse=lse, stream=stream)
            return self.out
        if append:
            nosa_pool_append(self.p, k_cache, v_cache, seq_start, seq_len, self.pooled,
                             max_new_keys=1, k_new=k_new, v_new=v_new, ws=self.ws, stream=stream)
        nosa_block_select(self.p, q, self.pooled, seq_len, self.max_seq_len, self.sel_idx,
                          self.sel_cnt, self.ws, stream=stream)
        nosa_sparse_decode(self.p, q, k_cache, v_cache, seq_start, seq_len, self.max_seq_len,
                           self.sel_idx, self.sel_cnt, self.out, self.ws, lse=lse, stream=stream)
        return self.out


def default_scale(head_dim: int = 128) -> float:
    return 1.0 / math.sqrt(head_dim)
