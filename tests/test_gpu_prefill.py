"""Sparse prefill (the NOSAS mode): every prefill token follows the decode
rule on its own prefix (L = position + 1).  GPU <-> oracle parity (B200),
and the multi-query launch against per-token decode launches."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from helpers import LSE_ATOL, assert_out_close, assert_valid_topk
from long_context_decode_nosa_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def nosa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_decode_nosa_b200 import build
    build.build()
    from long_context_decode_nosa_b200 import nosa as m
    m.lib()
    return m


def _status_ok(nosa, ws):
    rc, bits = nosa.nosa_read_device_status(ws)
    assert rc == 0 and bits == 0, (rc, hex(bits))


def _setup(nosa, lens, rows, hq, hkv, topk, seed, **pkw):
    """Caches of `lens` tokens; query rows (first position, count) per sequence;
    pooled keys of every window of each sequence (the prefill appends them
    before attending).  Returns host batch, device tensors and params."""
    b = inputs.make_batch(lens, num_q_heads=hq, num_kv_heads=hkv, seed=seed)
    q_pos = torch.tensor([r[0] for r in rows], dtype=torch.int32)
    q_start = torch.tensor(np.concatenate([[0], np.cumsum([r[1] for r in rows])]), dtype=torch.int32)
    total_q = int(q_start[-1])
    gen = torch.Generator().manual_seed(seed + 1)
    q = torch.randn(total_q, hq, 128, generator=gen).to(torch.bfloat16)
    p = nosa.params(hq, hkv, topk=topk, **pkw)
    g = b.to(DEV)
    if p.kv_int8:
        g.k_cache, g.v_cache = nosa.Int8KvCache.from_bf16(p, g.k_cache), nosa.Int8KvCache.from_bf16(p, g.v_cache)
    nc_cap = max(1, nosa.n_windows(max(lens)))
    pooled = torch.zeros(len(lens), hkv, nc_cap, 128, dtype=p.pooled_dtype, device=DEV)
    # the prefill's own pooling step: the windows before each chunk, then the
    # windows the chunk's rows complete
    ws = nosa.workspace(p, len(lens), max(lens))
    nosa.nosa_pool_append(p, g.k_cache, None, g.seq_start, q_pos.to(DEV), pooled,
                          len_old=torch.zeros_like(q_pos).to(DEV), max_new_keys=nc_cap, ws=ws)
    lens_end = (q_pos + (q_start[1:] - q_start[:-1])).to(torch.int32)
    nosa.nosa_pool_append(p, g.k_cache, None, g.seq_start, lens_end.to(DEV), pooled, len_old=q_pos.to(DEV),
                          max_new_keys=nc_cap, ws=ws)
    _status_ok(nosa, ws)
    return b, g, p, q, q_start, q_pos, pooled, total_q, lens_end


def _run(nosa, g, p, q, q_start, q_pos, pooled, total_q, max_len):
    hq, hkv = p.num_q_heads, p.num_kv_heads
    sel = torch.full((total_q, hkv, p.topk), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((total_q, hkv), -7, dtype=torch.int32, device=DEV)
    out = torch.empty(total_q, hq, 128, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(total_q, hq, device=DEV)
    ws = nosa.prefill_workspace(p, total_q, max_len)
    nosa.nosa_sparse_prefill(p, q.to(DEV), g.k_cache, g.v_cache, g.seq_start, q_start.to(DEV), q_pos.to(DEV),
                             max_len, pooled, sel, cnt, out, ws, lse=lse)
    torch.cuda.synchronize()
    _status_ok(nosa, ws)
    return sel, cnt, out, lse


@pytest.mark.parametrize("hq,hkv,topk", [(16, 2, 16), (32, 8, 8), (8, 8, 4), (64, 4, 8), (4, 2, 12)])
def test_sparse_prefill_matches_oracle(nosa, hq, hkv, topk):
    """Chunks at the start of a sequence, in its middle (crossing block and
    local-window boundaries) and a single row; ragged lengths; every group
    size (G = 8, 4, 1, 16, 2), so query groups of 8, 16, 64, 4 and 32 rows,
    some holding rows of two sequences."""
    lens = [3000, 2600, 1200]
    rows = [(2900, 100), (0, 130), (1100, 1)]
    b, g, p, q, q_start, q_pos, pooled, total_q, lens_end = _setup(nosa, lens, rows, hq, hkv, topk, seed=41 + hq)
    sel, cnt, out, lse = _run(nosa, g, p, q, q_start, q_pos, pooled, total_q, max(lens))
    ref_pooled = oracle.pool(inputs.bf16_bits(b.k_cache), b.seq_start.numpy(), lens_end.numpy(), pooled.shape[2])
    np.testing.assert_allclose(pooled.cpu().numpy(), ref_pooled, rtol=2e-6, atol=1e-6)
    rsel, rcnt, rout, rlse = oracle.sparse_prefill(inputs.bf16_bits(q), inputs.bf16_bits(b.k_cache),
                                                   inputs.bf16_bits(b.v_cache), b.seq_start.numpy(),
                                                   q_start.numpy(), q_pos.numpy(), ref_pooled, topk)
    sel_h, cnt_h = sel.cpu().numpy(), cnt.cpu().numpy()
    np.testing.assert_array_equal(cnt_h, rcnt)
    # selections valid against the oracle's block scores of each token's prefix
    same = (sel_h == rsel).all(axis=2)
    assert same.mean() > 0.9
    G = hq // hkv
    mask = np.repeat(same, G, axis=1)
    assert_out_close(out.float().cpu().numpy()[mask], rout[mask])
    np.testing.assert_allclose(lse.cpu().numpy()[mask], rlse[mask], atol=LSE_ATOL, rtol=0)
    # where the selections differ, they must be valid top-k sets of the oracle's scores
    for e, h in zip(*np.nonzero(~same)):
        s_ = int(np.searchsorted(q_start.numpy(), e, side="right") - 1)
        L = int(q_pos[s_]) + e - int(q_start[s_]) + 1
        sc = oracle.comp_scores(inputs.bf16_bits(q[e:e + 1]), ref_pooled[s_:s_ + 1], np.array([L], np.int32),
                                num_kv_heads=hkv)
        S = oracle.block_scores(sc, np.array([L], np.int32), oracle.n_blocks(L), num_kv_heads=hkv)
        nc = oracle.n_candidates(L)
        scale = np.max(np.abs(S[0, h, :nc])) if nc else 1.0
        assert_valid_topk(sel_h[e, h], cnt_h[e, h], S[0, h], nc, topk, 1e-5 * scale)


def test_sparse_prefill_dense_budget_is_causal_attention(nosa):
    """Top-k covering every candidate: each row attends to its whole prefix,
    so the GPU output is causal attention (torch fp64 SDPA, lower-triangular
    mask) within the attention tolerances."""
    lens = [2500]
    rows = [(2300, 200)]
    topk = 32
    b, g, p, q, q_start, q_pos, pooled, total_q, _ = _setup(nosa, lens, rows, 16, 2, topk, seed=45)
    assert topk >= nosa.n_blocks(2500) - 16
    sel, cnt, out, lse = _run(nosa, g, p, q, q_start, q_pos, pooled, total_q, 2500)
    k = b.k_cache[:2500].double().permute(1, 0, 2).repeat_interleave(8, 0)
    v = b.v_cache[:2500].double().permute(1, 0, 2).repeat_interleave(8, 0)
    qq = q.double().permute(1, 0, 2)
    m = torch.arange(2500)[None, :] <= (2300 + torch.arange(200))[:, None]
    o_ref = F.scaled_dot_product_attention(qq, k, v, attn_mask=m).permute(1, 0, 2).numpy()
    assert_out_close(out.float().cpu().numpy(), o_ref)
    logits = (qq @ k.transpose(-1, -2)) / math.sqrt(128)
    l_ref = torch.logsumexp(logits.masked_fill(~m, -math.inf), dim=-1).t().numpy()
    np.testing.assert_allclose(lse.cpu().numpy(), l_ref, atol=LSE_ATOL, rtol=0)


@pytest.mark.parametrize("kv_int8", [False, True])
def test_sparse_prefill_equals_per_token_decode(nosa, kv_int8):
    """The multi-query launch gives what block_select + sparse_decode give for
    each token with L = position + 1 (bf16 and INT8 caches): the same
    selection bit for bit, the same attention up to rounding -- the cluster
    size depends on how many entries a launch holds, and with another split
    of the tiles each CTA's running maximum, and so the bf16 rounding of its
    softmax weights, differs (about 2^-9 of a weight)."""
    lens = [5000, 3000]
    rows = [(4900, 70), (2000, 33)]
    b, g, p, q, q_start, q_pos, pooled, total_q, _ = _setup(nosa, lens, rows, 16, 2, 64, seed=47, kv_int8=kv_int8)
    sel, cnt, out, lse = _run(nosa, g, p, q, q_start, q_pos, pooled, total_q, max(lens))
    qd = q.to(DEV)
    for s_, (p0, n) in enumerate(rows):
        e0 = int(q_start[s_])
        L = torch.arange(p0 + 1, p0 + n + 1, dtype=torch.int32, device=DEV)
        st = torch.full((n,), int(b.seq_start[s_]), dtype=torch.int64, device=DEV)
        pl = pooled[s_:s_ + 1].expand(n, -1, -1, -1).contiguous()
        sel1 = torch.empty(n, 2, 64, dtype=torch.int32, device=DEV)
        cnt1 = torch.empty(n, 2, dtype=torch.int32, device=DEV)
        out1 = torch.empty(n, 16, 128, dtype=torch.bfloat16, device=DEV)
        lse1 = torch.empty(n, 16, device=DEV)
        ws = nosa.workspace(p, n, max(lens))
        nosa.nosa_block_select(p, qd[e0:e0 + n], pl, L, max(lens), sel1, cnt1, ws)
        nosa.nosa_sparse_decode(p, qd[e0:e0 + n], g.k_cache, g.v_cache, st, L, max(lens), sel1, cnt1, out1, ws,
                                lse=lse1)
        torch.cuda.synchronize()
        _status_ok(nosa, ws)
        assert torch.equal(sel1, sel[e0:e0 + n]) and torch.equal(cnt1, cnt[e0:e0 + n])
        torch.testing.assert_close(out1.float(), out[e0:e0 + n].float(), rtol=1e-2, atol=5e-4)
        torch.testing.assert_close(lse1, lse[e0:e0 + n], rtol=0, atol=1e-5)


def test_sparse_prefill_reports_rows_past_max_len(nosa):
    lens = [1500]
    rows = [(1400, 100)]
    b, g, p, q, q_start, q_pos, pooled, total_q, _ = _setup(nosa, lens, rows, 16, 2, 8, seed=49)
    ws = nosa.prefill_workspace(p, total_q, 1450)
    sel = torch.empty(total_q, 2, 8, dtype=torch.int32, device=DEV)
    cnt = torch.empty(total_q, 2, dtype=torch.int32, device=DEV)
    out = torch.empty(total_q, 16, 128, dtype=torch.bfloat16, device=DEV)
    nosa.nosa_sparse_prefill(p, q.to(DEV), g.k_cache, g.v_cache, g.seq_start, q_start.to(DEV), q_pos.to(DEV), 1450,
                             pooled, sel, cnt, out, ws)
    rc, bits = nosa.nosa_read_device_status(ws)
    assert rc == nosa.NOSA_ERR_DEVICE_CHECK and bits & nosa.NOSA_DEV_MAX_LEN
    assert (cnt[50:] == 0).all() and torch.isfinite(out.float()).all()


@pytest.mark.parametrize("kv_int8", [False, True])
def test_sparse_prefill_paged_equals_contiguous(nosa, kv_int8):
    """The same tokens in shuffled 64-token pages: selection, output and lse
    bit-identical to the contiguous call (bf16 caches: grouped attention;
    INT8: per-entry attention)."""
    lens = [3000, 2600, 1200]
    rows = [(2900, 100), (0, 130), (1100, 1)]
    b, g, p, q, q_start, q_pos, pooled, total_q, _ = _setup(nosa, lens, rows, 16, 2, 16, seed=51, kv_int8=kv_int8)
    sel, cnt, out, lse = _run(nosa, g, p, q, q_start, q_pos, pooled, total_q, max(lens))
    # pages of the bf16 caches, quantized afresh for INT8 (same codes: per-row quantization)
    cap = b.capacity.numpy()
    need = [(int(c) + 63) // 64 for c in cap]
    num_pages = sum(need) + 3
    perm = np.random.default_rng(52).permutation(num_pages)
    table = np.full((b.batch, max(need)), -1, np.int32)
    src, dst, n = [], [], 0
    for i in range(b.batch):
        for pg in range(need[i]):
            table[i, pg] = perm[n]
            n += 1
            t = np.arange(pg * 64, min(pg * 64 + 64, int(cap[i])))
            src.append(int(b.seq_start[i]) + t)
            dst.append(int(table[i, pg]) * 64 + t - pg * 64)
    src = torch.from_numpy(np.concatenate(src)).to(DEV)
    dst = torch.from_numpy(np.concatenate(dst)).to(DEV)
    kb, vb = b.k_cache.to(DEV), b.v_cache.to(DEV)
    kp = torch.zeros(num_pages * 64, 2, 128, dtype=torch.bfloat16, device=DEV)
    vp = torch.zeros_like(kp)
    kp[dst] = kb[src]
    vp[dst] = vb[src]
    if kv_int8:
        kp, vp = nosa.Int8KvCache.from_bf16(p, kp), nosa.Int8KvCache.from_bf16(p, vp)
    table_d = torch.from_numpy(table).to(DEV)
    sel2 = torch.full_like(sel, -7)
    cnt2 = torch.full_like(cnt, -7)
    out2 = torch.empty_like(out)
    lse2 = torch.empty_like(lse)
    ws = nosa.prefill_workspace(p, total_q, max(lens))
    nosa.nosa_sparse_prefill_paged(p, q.to(DEV), kp, vp, table_d, q_start.to(DEV), q_pos.to(DEV), max(lens), pooled,
                                   sel2, cnt2, out2, ws, lse=lse2)
    torch.cuda.synchronize()
    _status_ok(nosa, ws)
    assert torch.equal(sel, sel2) and torch.equal(cnt, cnt2)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_sparse_prefill_tcgen05_kernel_passes_the_same_tests():
    """The tcgen05 (TMEM-accumulator) attention kernel, selected with
    NOSA_PREFILL_UMMA=1 (read once per process), passes this file's parity
    tests in a child process."""
    import os
    import subprocess
    import sys
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, NOSA_PREFILL_UMMA="1")
    here = os.path.dirname(os.path.abspath(__file__))
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(here, "test_gpu_prefill.py"), "-x", "-q",
                        "-m", "gpu", "-k", "not tcgen05"], env=env, cwd=os.path.dirname(here),
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
