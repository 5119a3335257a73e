"""Shared test helpers: run the CPU oracle on a DecodeBatch, compare results."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from long_context_decode_nosa_b200 import inputs

# Tolerances (written here once, used by every parity test):
#   compressed / block scores: |gpu - ref| <= 1e-3 * max(|ref|, 1e-3 * max|ref row|)
#   attention output (bf16 out, fp32 accumulate): |gpu - ref| <= 2e-2 + 1e-2 * |ref|
#   lse: |gpu - ref| <= 1e-3
SCORE_RTOL = 1e-3
OUT_ATOL, OUT_RTOL = 2e-2, 1e-2
LSE_ATOL = 1e-3


def sub_batch(b: inputs.DecodeBatch, seqs) -> inputs.DecodeBatch:
    """The listed sequences of ``b`` as their own host batch (K/V rows copied)."""
    seqs = list(seqs)
    lens = [int(b.seq_len[i]) for i in seqs]
    starts, rows_k, rows_v, off = [], [], [], 0
    for i in seqs:
        s0, L = int(b.seq_start[i]), int(b.seq_len[i])
        rows_k.append(b.k_cache[s0:s0 + L].cpu())
        rows_v.append(b.v_cache[s0:s0 + L].cpu())
        starts.append(off)
        off += L
    return inputs.DecodeBatch(b.q[seqs].cpu(), torch.cat(rows_k), torch.cat(rows_v),
                              torch.tensor(starts, dtype=torch.int64),
                              torch.tensor(lens, dtype=torch.int32),
                              torch.tensor(lens, dtype=torch.int32),
                              b.num_q_heads, b.num_kv_heads, b.head_dim)


def oracle_int8_caches(b: inputs.DecodeBatch):
    """The oracle's own INT8 quantization of b's caches: (k_codes, k_scales,
    v_codes, v_scales), scales [T, Hkv]."""
    kc, ks = oracle.quantize_int8(inputs.bf16_bits(b.k_cache))
    vc, vs = oracle.quantize_int8(inputs.bf16_bits(b.v_cache))
    return kc, ks, vc, vs


def oracle_step(b: inputs.DecodeBatch, topk: int, *, local_blocks: int = 16, scale=None, pooled_bf16=False,
                kv_int8=None):
    """Pool every window, then the whole selection + attention, on the oracle.
    ``kv_int8``: the caches as (k_codes, k_scales, v_codes, v_scales) (the
    INT8 cache variant) instead of b's bf16 caches."""
    kb = inputs.bf16_bits(b.k_cache)
    lens = b.seq_len.cpu().numpy()
    nc_cap = max(1, oracle.n_windows(int(lens.max())))
    if kv_int8 is not None:
        kc, ks, vc, vs = kv_int8
        pooled = oracle.pool_int8(kc, ks, b.seq_start.cpu().numpy(), lens, nc_cap, bf16=pooled_bf16)
    else:
        pooled = oracle.pool(kb, b.seq_start.cpu().numpy(), lens, nc_cap, bf16=pooled_bf16)
    nb_cap = oracle.n_blocks(int(lens.max()))
    s = oracle.comp_scores(inputs.bf16_bits(b.q), pooled, lens, num_kv_heads=b.num_kv_heads,
                           scale=scale)
    S = oracle.block_scores(s, lens, nb_cap, num_kv_heads=b.num_kv_heads,
                            local_blocks=local_blocks)
    idx, cnt = oracle.topk(S, lens, topk, local_blocks=local_blocks)
    if kv_int8 is not None:
        out, lse = oracle.sparse_attention_int8(inputs.bf16_bits(b.q), kc, ks, vc, vs, b.seq_start.cpu().numpy(),
                                                lens, idx, cnt, scale=scale, local_blocks=local_blocks)
    else:
        out, lse = oracle.sparse_attention(inputs.bf16_bits(b.q), kb, inputs.bf16_bits(b.v_cache),
                                           b.seq_start.cpu().numpy(), lens, idx, cnt, scale=scale,
                                           local_blocks=local_blocks)
    return dict(pooled=pooled, comp_scores=s, block_scores=S, sel_idx=idx, sel_cnt=cnt, out=out,
                lse=lse)


def assert_scores_close(gpu, ref, valid_mask=None):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    if valid_mask is None:
        valid_mask = np.isfinite(ref)
    g, r = gpu[valid_mask], ref[valid_mask]
    if r.size == 0:
        return
    floor = 1e-3 * np.max(np.abs(r))
    tol = SCORE_RTOL * np.maximum(np.abs(r), floor)
    bad = np.abs(g - r) > tol
    assert not bad.any(), f"{bad.sum()} of {r.size} scores off; worst {np.max(np.abs(g - r) - tol)}"


def assert_out_close(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref) - (OUT_ATOL + OUT_RTOL * np.abs(ref))
    assert (err <= 0).all(), f"{(err > 0).sum()} outputs off; worst excess {err.max()}"


def assert_valid_topk(sel, cnt, S_ref, ncand, topk, tol):
    """GPU selection vs the oracle's block scores: exactly min(topk, ncand)
    distinct ascending candidates; every block scoring above the k-th score by
    more than ``tol`` is in, every block below it by more than ``tol`` is out."""
    k = min(topk, ncand)
    assert cnt == k
    chosen = [int(x) for x in sel[:k]]
    assert chosen == sorted(set(chosen)) and all(0 <= c < ncand for c in chosen)
    assert all(int(x) == -1 for x in sel[k:])
    if k == 0 or k == ncand:
        assert chosen == list(range(ncand))[:k] if k == ncand else True
        return
    sc = np.asarray(S_ref[:ncand], np.float64)
    kth = np.sort(sc)[::-1][k - 1]
    must = set(np.nonzero(sc > kth + tol)[0].tolist())
    never = set(np.nonzero(sc < kth - tol)[0].tolist())
    cs = set(chosen)
    assert must <= cs, sorted(must - cs)
    assert not (never & cs), sorted(never & cs)
