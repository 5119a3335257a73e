"""CPU oracle for NOSA sparse decode attention -- TEST INFRASTRUCTURE.

Only the test-suite (``tests/``), ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library and its Python binding never import it; the two
share no code.

The arithmetic lives in ``nosa_oracle.c`` (plain C loops, fp64 sums, one
rounding to fp32 per pooled key / score, as documented there).  This module
only marshals numpy arrays through ctypes.  bf16 tensors travel as their
16-bit patterns (``uint16``).

Every function is pinned by ``tests/test_oracle_pins.py`` against closed forms,
brute force on tiny inputs and a library attention routine.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from .build import LIB, build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            _build()
        lib = ctypes.CDLL(LIB)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.nosa_oracle_set_threads.argtypes = [i32]
        lib.nosa_oracle_set_threads.restype = i32
        lib.nosa_oracle_pool.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, P, i64]
        lib.nosa_oracle_comp_scores.argtypes = [P, P, i64, P, i32, i32, i32, i32, i32, i32, f64, P]
        lib.nosa_oracle_block_scores.argtypes = [P, i64, P, i32, i32, i32, i32, i32, i32, i32, P, i64]
        lib.nosa_oracle_topk.argtypes = [P, i64, P, i32, i32, i32, i32, i32, P, P]
        lib.nosa_oracle_sparse_attention.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32,
                                                     P, P, i32, f64, P, P]
        lib.nosa_oracle_quantize_int8.argtypes = [P, i64, i32, P, P]
        lib.nosa_oracle_pool_int8.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, P, i64]
        lib.nosa_oracle_sparse_attention_int8.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                                          i32, P, P, i32, f64, P, P]
        for name in ("nosa_oracle_pool", "nosa_oracle_comp_scores", "nosa_oracle_block_scores",
                     "nosa_oracle_topk", "nosa_oracle_sparse_attention", "nosa_oracle_quantize_int8",
                     "nosa_oracle_pool_int8", "nosa_oracle_sparse_attention_int8"):
            getattr(lib, name).restype = i32
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: oracle rejected its arguments (code {rc})")


def set_threads(n: int) -> int:
    """OpenMP threads for loops over independent (sequence, KV head) pairs."""
    return _load().nosa_oracle_set_threads(int(n))


def n_windows(L: int, kernel: int = 32, stride: int = 16) -> int:
    return (L - kernel) // stride + 1 if L >= kernel else 0


def n_blocks(L: int, bs: int = 64) -> int:
    return (L + bs - 1) // bs


def n_candidates(L: int, bs: int = 64, local_blocks: int = 16) -> int:
    return max(0, n_blocks(L, bs) - local_blocks)


def round_bf16(x):
    """fp32 values rounded to the nearest bfloat16, ties to even, returned as
    fp32 (the bf16 pooled-key variant keeps its pooled keys this way).  On the
    fp32 bit pattern: add 0x7FFF plus the lowest kept bit, then clear the 16
    dropped bits; NaN stays NaN, infinities stay infinite, and finite values
    past the largest bf16 round to infinity."""
    x = np.asarray(x, np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    out = r.view(np.float32).copy()
    out[np.isnan(x)] = np.nan
    return out


def pool(k_cache, seq_start, len_new, nc_cap, *, len_old=None, pooled=None,
         kernel=32, stride=16, bf16=False):
    """Mean-pooled keys: windows [nc(len_old), nc(len_new)) of every (seq, KV head).

    k_cache: uint16 [T, Hkv, D] (bf16 bits).  Returns fp32 [B, Hkv, nc_cap, D];
    windows that were not (re)computed keep the contents of ``pooled`` (zeros
    when ``pooled`` is None).  ``bf16``: every pooled key rounded to bfloat16
    (round_bf16), the bf16 pooled-key variant."""
    k_cache = _c(k_cache, np.uint16)
    T, hkv, d = k_cache.shape
    seq_start = _c(seq_start, np.int64)
    len_new = _c(len_new, np.int32)
    B = len_new.shape[0]
    len_old = None if len_old is None else _c(len_old, np.int32)
    out = np.zeros((B, hkv, nc_cap, d), np.float32) if pooled is None else _c(pooled, np.float32).copy()
    rc = _load().nosa_oracle_pool(_ptr(k_cache), _ptr(seq_start), _ptr(len_old), _ptr(len_new),
                                  B, hkv, d, kernel, stride, _ptr(out), nc_cap)
    _check(rc, "pool")
    return round_bf16(out) if bf16 else out


def quantize_int8(x):
    """INT8 cache variant: rows of bf16 values (uint16 bits, [..., d]) to
    (codes int8 [..., d], scales fp32 [...]), symmetric per row:
    s = max|x| / 127, code = clamp(rint(x / s), -127, 127) in fp32, half to
    even; s = 0 and zero codes for an all-zero row."""
    x = _c(x, np.uint16)
    d = x.shape[-1]
    rows = x.size // d
    codes = np.empty(x.shape, np.int8)
    scales = np.empty(x.shape[:-1], np.float32)
    rc = _load().nosa_oracle_quantize_int8(_ptr(x), rows, d, _ptr(codes), _ptr(scales))
    _check(rc, "quantize_int8")
    return codes, scales


def pool_int8(k_codes, k_scales, seq_start, len_new, nc_cap, *, len_old=None, pooled=None,
              kernel=32, stride=16, bf16=False):
    """``pool`` over an INT8 key cache: codes int8 [T, Hkv, D], scales fp32
    [T, Hkv]; each window's mean of the dequantized keys s_t * code_t."""
    k_codes = _c(k_codes, np.int8)
    k_scales = _c(k_scales, np.float32)
    T, hkv, d = k_codes.shape
    assert k_scales.shape == (T, hkv)
    seq_start = _c(seq_start, np.int64)
    len_new = _c(len_new, np.int32)
    B = len_new.shape[0]
    len_old = None if len_old is None else _c(len_old, np.int32)
    out = np.zeros((B, hkv, nc_cap, d), np.float32) if pooled is None else _c(pooled, np.float32).copy()
    rc = _load().nosa_oracle_pool_int8(_ptr(k_codes), _ptr(k_scales), _ptr(seq_start), _ptr(len_old),
                                       _ptr(len_new), B, hkv, d, kernel, stride, _ptr(out), nc_cap)
    _check(rc, "pool_int8")
    return round_bf16(out) if bf16 else out


def comp_scores(q, pooled, seq_len, *, num_kv_heads, scale=None, kernel=32, stride=16):
    """Compressed scores s[B, Hq, nc_cap] fp32 (-inf past nc(L_i))."""
    q = _c(q, np.uint16)
    B, hq, d = q.shape
    pooled = _c(pooled, np.float32)
    nc_cap = pooled.shape[2]
    seq_len = _c(seq_len, np.int32)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    s = np.empty((B, hq, nc_cap), np.float32)
    rc = _load().nosa_oracle_comp_scores(_ptr(q), _ptr(pooled), nc_cap, _ptr(seq_len), B, hq,
                                         num_kv_heads, d, kernel, stride, scale, _ptr(s))
    _check(rc, "comp_scores")
    return s


def block_scores(s, seq_len, nb_cap, *, num_kv_heads, kernel=32, stride=16, block_size=64,
                 local_blocks=16):
    """Block scores S[B, Hkv, nb_cap] fp32 (-inf for non-candidates)."""
    s = _c(s, np.float32)
    B, hq, nc_cap = s.shape
    seq_len = _c(seq_len, np.int32)
    S = np.empty((B, num_kv_heads, nb_cap), np.float32)
    rc = _load().nosa_oracle_block_scores(_ptr(s), nc_cap, _ptr(seq_len), B, hq, num_kv_heads,
                                          kernel, stride, block_size, local_blocks, _ptr(S), nb_cap)
    _check(rc, "block_scores")
    return S


def topk(S, seq_len, topk, *, block_size=64, local_blocks=16):
    """(sel_idx int32 [B, Hkv, topk] ascending, -1 padded; sel_cnt int32 [B, Hkv])."""
    S = _c(S, np.float32)
    B, hkv, nb_cap = S.shape
    seq_len = _c(seq_len, np.int32)
    idx = np.empty((B, hkv, topk), np.int32)
    cnt = np.empty((B, hkv), np.int32)
    rc = _load().nosa_oracle_topk(_ptr(S), nb_cap, _ptr(seq_len), B, hkv, block_size,
                                  local_blocks, topk, _ptr(idx), _ptr(cnt))
    _check(rc, "topk")
    return idx, cnt


def sparse_attention(q, k_cache, v_cache, seq_start, seq_len, sel_idx, sel_cnt, *, scale=None,
                     block_size=64, local_blocks=16):
    """Attention over selected blocks + local window: (out fp64 [B,Hq,D], lse fp64 [B,Hq])."""
    q = _c(q, np.uint16)
    B, hq, d = q.shape
    k_cache = _c(k_cache, np.uint16)
    v_cache = _c(v_cache, np.uint16)
    hkv = k_cache.shape[1]
    sel_idx = _c(sel_idx, np.int32)
    sel_cnt = _c(sel_cnt, np.int32)
    tk = sel_idx.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = np.empty((B, hq, d), np.float64)
    lse = np.empty((B, hq), np.float64)
    rc = _load().nosa_oracle_sparse_attention(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(_c(seq_start, np.int64)),
        _ptr(_c(seq_len, np.int32)), B, hq, hkv, d, block_size, local_blocks,
        _ptr(sel_idx), _ptr(sel_cnt), tk, scale, _ptr(out), _ptr(lse))
    _check(rc, "sparse_attention")
    return out, lse


def sparse_attention_int8(q, k_codes, k_scales, v_codes, v_scales, seq_start, seq_len, sel_idx, sel_cnt, *,
                          scale=None, block_size=64, local_blocks=16):
    """``sparse_attention`` over INT8 caches (codes int8 [T, Hkv, D], scales
    fp32 [T, Hkv]): keys and values are s_t * code_t."""
    q = _c(q, np.uint16)
    B, hq, d = q.shape
    k_codes, v_codes = _c(k_codes, np.int8), _c(v_codes, np.int8)
    k_scales, v_scales = _c(k_scales, np.float32), _c(v_scales, np.float32)
    hkv = k_codes.shape[1]
    sel_idx = _c(sel_idx, np.int32)
    sel_cnt = _c(sel_cnt, np.int32)
    tk = sel_idx.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = np.empty((B, hq, d), np.float64)
    lse = np.empty((B, hq), np.float64)
    rc = _load().nosa_oracle_sparse_attention_int8(
        _ptr(q), _ptr(k_codes), _ptr(k_scales), _ptr(v_codes), _ptr(v_scales),
        _ptr(_c(seq_start, np.int64)), _ptr(_c(seq_len, np.int32)), B, hq, hkv, d, block_size,
        local_blocks, _ptr(sel_idx), _ptr(sel_cnt), tk, scale, _ptr(out), _ptr(lse))
    _check(rc, "sparse_attention_int8")
    return out, lse


def decode_step(q, k_cache, v_cache, seq_start, seq_len, pooled, topk_blocks, *, scale=None,
                kernel=32, stride=16, block_size=64, local_blocks=16):
    """The whole per-step path in the pages' order: compressed scores -> block
    scores -> top-k -> exact attention.  ``pooled`` must already hold the
    pooled keys of [0, nc(L_i)).  Returns a dict of every intermediate."""
    hkv = k_cache.shape[1]
    nb_cap = n_blocks(int(np.max(seq_len)), block_size)
    s = comp_scores(q, pooled, seq_len, num_kv_heads=hkv, scale=scale, kernel=kernel, stride=stride)
    S = block_scores(s, seq_len, nb_cap, num_kv_heads=hkv, kernel=kernel, stride=stride,
                     block_size=block_size, local_blocks=local_blocks)
    idx, cnt = topk(S, seq_len, topk_blocks, block_size=block_size, local_blocks=local_blocks)
    out, lse = sparse_attention(q, k_cache, v_cache, seq_start, seq_len, idx, cnt, scale=scale,
                                block_size=block_size, local_blocks=local_blocks)
    return {"comp_scores": s, "block_scores": S, "sel_idx": idx, "sel_cnt": cnt,
            "out": out, "lse": lse}


def sparse_prefill(q, k_cache, v_cache, seq_start, q_start, q_pos, pooled, topk_blocks, *, scale=None,
                   kernel=32, stride=16, block_size=64, local_blocks=16):
    """Sparse prefill (the NOSAS mode): every query row e of sequence s (rows
    q_start[s] .. q_start[s+1]-1, positions q_pos[s] + r) is one decode step
    of its own prefix, L = position + 1, against sequence s's cache and
    pooled keys -- ``decode_step`` applied token by token.  ``pooled``
    [batch, Hkv, nc_cap, D] must hold every window of each prefix.  Returns
    (sel_idx [total_q, Hkv, topk], sel_cnt [total_q, Hkv], out fp64
    [total_q, Hq, D], lse fp64 [total_q, Hq])."""
    q = _c(q, np.uint16)
    total_q, hq, d = q.shape
    hkv = k_cache.shape[1]
    q_start = np.asarray(q_start, np.int64)
    q_pos = np.asarray(q_pos, np.int64)
    seq_start = np.asarray(seq_start, np.int64)
    sel = np.full((total_q, hkv, topk_blocks), -1, np.int32)
    cnt = np.zeros((total_q, hkv), np.int32)
    out = np.zeros((total_q, hq, d), np.float64)
    lse = np.zeros((total_q, hq), np.float64)
    for s_ in range(len(q_pos)):
        for e in range(int(q_start[s_]), int(q_start[s_ + 1])):
            L = int(q_pos[s_]) + (e - int(q_start[s_])) + 1
            r = decode_step(q[e:e + 1], k_cache, v_cache, seq_start[s_:s_ + 1], np.array([L], np.int32),
                            pooled[s_:s_ + 1], topk_blocks, scale=scale, kernel=kernel, stride=stride,
                            block_size=block_size, local_blocks=local_blocks)
            sel[e], cnt[e], out[e], lse[e] = r["sel_idx"][0], r["sel_cnt"][0], r["out"][0], r["lse"][0]
    return sel, cnt, out, lse
