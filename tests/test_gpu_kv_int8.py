"""INT8 K/V caches (nosa_params.kv_int8): GPU <-> oracle parity (B200).

The quantizer is compared bit for bit with the oracle's (same fp32
divisions, half-to-even rounding).  Everything downstream runs each side on
its own quantized caches: pooling within fp32 summation error of the
oracle's fp64 mean of s * code, attention within the usual tolerances of the
oracle's attention over s * code, the fused step bit-identical to the
separate launches and the paged layout bit-identical to the contiguous one."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from helpers import LSE_ATOL, assert_out_close, assert_valid_topk, oracle_int8_caches, oracle_step
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


def _quantized(nosa, p, g):
    return nosa.Int8KvCache.from_bf16(p, g.k_cache), nosa.Int8KvCache.from_bf16(p, g.v_cache)


def test_quantize_matches_oracle_bit_for_bit(nosa):
    """Gaussian rows over 40 binades, all-zero rows, exact halfway values and
    a ragged row count (scale stride padding)."""
    rng = np.random.default_rng(81)
    rows, hkv = 4099, 2
    x = rng.standard_normal((rows, hkv, 128)) * np.exp(rng.uniform(-20, 20, (rows, hkv, 1)))
    x[5] = 0.0
    x[7, 1] = np.concatenate([[127.0], np.arange(127) + 0.5]) * 2.0 ** -3
    src = torch.from_numpy(x).to(torch.bfloat16)
    p = nosa.params(16, hkv, kv_int8=True)
    c = nosa.Int8KvCache.from_bf16(p, src.to(DEV))
    torch.cuda.synchronize()
    codes, scales = oracle.quantize_int8(inputs.bf16_bits(src))
    np.testing.assert_array_equal(c.codes.cpu().numpy(), codes)
    np.testing.assert_array_equal(c.row_scales().cpu().numpy().view(np.uint32), scales.view(np.uint32))
    # a row range into an existing buffer leaves the other rows alone
    part = nosa.Int8KvCache(rows, hkv)
    nosa.nosa_quantize_kv_int8(p, src[100:300].to(DEV), part, row0=100)
    torch.cuda.synchronize()
    got = part.codes.cpu().numpy()
    np.testing.assert_array_equal(got[100:300], codes[100:300])
    assert not got[:100].any() and not got[300:].any()


def test_pool_int8_matches_oracle(nosa):
    lens = [16384, 5000, 33, 31, 700]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=82)
    g = b.to(DEV)
    p = nosa.params(16, 2, kv_int8=True)
    kq, _ = _quantized(nosa, p, g)
    st = nosa.DecodeState(p, b.batch, max(lens))
    st.rebuild_pooled(kq, g.seq_start, g.seq_len)
    kc, ks, _, _ = oracle_int8_caches(b)
    ref = oracle.pool_int8(kc, ks, b.seq_start.numpy(), b.seq_len.numpy(), st.nc_cap)
    got = st.pooled.cpu().numpy()
    v = np.abs(kc.astype(np.float64) * ks.astype(np.float64)[..., None])
    for i, L in enumerate(lens):
        nc = oracle.n_windows(L)
        s0 = int(b.seq_start[i])
        for j in range(nc):
            bound = 2.0 ** -21 * v[s0 + 16 * j:s0 + 16 * j + 32].sum(axis=0) / 32 + 1e-38   # [Hkv, D]
            assert (np.abs(got[i, :, j] - ref[i, :, j]) <= bound).all(), (i, j)
    _status_ok(nosa, st.ws)


def test_append_int8_equals_rebuild_and_oracle_quantizer(nosa):
    """Forty single-token appends (the rows quantized on the way in) give the
    rebuild's pooled bits; the appended codes and scales are the oracle's."""
    lens = [4096 + 40, 3000]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=83, slack=64).to(DEV)
    p = nosa.params(16, 2, kv_int8=True)
    kq, vq = _quantized(nosa, p, b)
    st = nosa.DecodeState(p, b.batch, max(lens) + 80)
    st.rebuild_pooled(kq, b.seq_start, b.seq_len)
    new_k, new_v = [], []
    for step in range(40):
        kn, vn = inputs.random_kv_rows(b.batch, 2, 128, seed=800 + step, device=DEV)
        new_k.append(kn.cpu())
        new_v.append(vn.cpu())
        b.seq_len += 1
        nosa.nosa_pool_append(p, kq, vq, b.seq_start, b.seq_len, st.pooled, max_new_keys=1, k_new=kn, v_new=vn,
                              ws=st.ws)
    inc = st.pooled.clone()
    st.pooled.zero_()
    st.rebuild_pooled(kq, b.seq_start, b.seq_len)
    assert torch.equal(inc, st.pooled)
    _status_ok(nosa, st.ws)
    starts = b.seq_start.cpu().numpy()
    for which, cache, rows in (("k", kq, new_k), ("v", vq, new_v)):
        codes, scales = oracle.quantize_int8(inputs.bf16_bits(torch.stack(rows)))   # [40, B, Hkv, D]
        got_c = cache.codes.cpu().numpy()
        got_s = cache.row_scales().cpu().numpy()
        for i, L in enumerate(lens):
            r = starts[i] + L + np.arange(40)
            np.testing.assert_array_equal(got_c[r], codes[:, i], err_msg=which)
            np.testing.assert_array_equal(got_s[r], scales[:, i], err_msg=which)


@pytest.mark.parametrize("hq,hkv,topk", [(16, 2, 64), (32, 8, 32), (8, 8, 16), (64, 4, 48)])
def test_sparse_decode_int8_matches_oracle(nosa, hq, hkv, topk):
    """Attention alone, on the oracle's selection: tiles with ragged tails,
    odd tile counts per CTA (one-tile jobs), every group size."""
    lens = [16384 + 37, 9000, 64 * 17 + 5, 700, 2049]
    b = inputs.make_batch(lens, num_q_heads=hq, num_kv_heads=hkv, seed=84 + hq)
    q8 = oracle_int8_caches(b)
    ref = oracle_step(b, topk, kv_int8=q8)
    g = b.to(DEV)
    p = nosa.params(hq, hkv, topk=topk, kv_int8=True)
    kq, vq = _quantized(nosa, p, g)
    ws = nosa.workspace(p, b.batch, max(lens))
    out = torch.empty(b.batch, hq, 128, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(b.batch, hq, device=DEV)
    nosa.nosa_sparse_decode(p, g.q, kq, vq, g.seq_start, g.seq_len, max(lens),
                            torch.from_numpy(ref["sel_idx"]).to(DEV), torch.from_numpy(ref["sel_cnt"]).to(DEV),
                            out, ws, lse=lse)
    torch.cuda.synchronize()
    assert_out_close(out.float().cpu().numpy(), ref["out"])
    np.testing.assert_allclose(lse.cpu().numpy(), ref["lse"], atol=LSE_ATOL, rtol=0)
    _status_ok(nosa, ws)


def test_dense_int8_window_only_and_zero_rows(nosa):
    """Sequences inside the local window (dense attention over s * code), a
    sequence whose cache rows are all zero (scale 0: uniform weights, zero
    output) and one of a single token."""
    lens = [1000, 64, 1, 300]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=85)
    s3 = int(b.seq_start[3])
    b.k_cache[s3:s3 + 300] = 0
    b.v_cache[s3:s3 + 300] = 0
    q8 = oracle_int8_caches(b)
    ref = oracle_step(b, 8, kv_int8=q8)
    g = b.to(DEV)
    p = nosa.params(16, 2, topk=8, kv_int8=True)
    kq, vq = _quantized(nosa, p, g)
    st = nosa.DecodeState(p, b.batch, max(lens))
    st.rebuild_pooled(kq, g.seq_start, g.seq_len)
    st.step(g.q, kq, vq, g.seq_start, g.seq_len, append=False, with_lse=True)
    torch.cuda.synchronize()
    assert_out_close(st.out.float().cpu().numpy(), ref["out"])
    np.testing.assert_allclose(st.lse.cpu().numpy(), ref["lse"], atol=LSE_ATOL, rtol=0)
    assert (st.out[3] == 0).all()
    _status_ok(nosa, st.ws)


def test_full_step_int8_matches_oracle(nosa):
    lens = [16384, 12000, 3000, 1100, 64 * 17 + 9, 40]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=86)
    q8 = oracle_int8_caches(b)
    ref = oracle_step(b, 64, kv_int8=q8)
    g = b.to(DEV)
    p = nosa.params(16, 2, topk=64, kv_int8=True)
    kq, vq = _quantized(nosa, p, g)
    st = nosa.DecodeState(p, b.batch, max(lens))
    st.rebuild_pooled(kq, g.seq_start, g.seq_len)
    st.step(g.q, kq, vq, g.seq_start, g.seq_len, append=False, with_lse=True)
    sel, cnt = st.sel_idx.cpu().numpy(), st.sel_cnt.cpu().numpy()
    for i, L in enumerate(lens):
        nc = oracle.n_candidates(L)
        for h in range(2):
            scale = np.max(np.abs(ref["block_scores"][i, h, :nc])) if nc else 1.0
            assert_valid_topk(sel[i, h], cnt[i, h], ref["block_scores"][i, h], nc, 64, 1e-5 * scale)
    same = (sel == ref["sel_idx"]).all(axis=2)
    mask = np.repeat(same, 8, axis=1)
    assert same.mean() > 0.5
    assert_out_close(st.out.float().cpu().numpy()[mask], ref["out"][mask])
    _status_ok(nosa, st.ws)


@pytest.mark.parametrize("pooled_bf16", [False, True])
def test_fused_step_int8_equals_separate_launches(nosa, pooled_bf16):
    lens = [16384, 7000, 2500, 16384, 64 * 20]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=87, slack=16)
    kn, vn = inputs.random_kv_rows(len(lens), 2, 128, seed=88)
    runs = []
    for fused in (True, False):
        g = b.to(DEV)
        p = nosa.params(16, 2, topk=64, kv_int8=True, pooled_bf16=pooled_bf16)
        kq, vq = _quantized(nosa, p, g)
        st = nosa.DecodeState(p, b.batch, max(lens) + 1)
        st.rebuild_pooled(kq, g.seq_start, g.seq_len)
        g.seq_len += 1
        st.step(g.q, kq, vq, g.seq_start, g.seq_len, fused=fused, with_lse=True, k_new=kn.to(DEV), v_new=vn.to(DEV))
        torch.cuda.synchronize()
        runs.append((st.out.clone(), st.lse.clone(), st.sel_idx.clone(), st.pooled.clone(), kq.buffer.clone(),
                     vq.buffer.clone()))
        _status_ok(nosa, st.ws)
    for x, y in zip(runs[0], runs[1]):
        assert torch.equal(x, y)


def test_paged_int8_equals_contiguous(nosa):
    """The same tokens in shuffled 64-token pages of an INT8 cache: pooling and
    the fused step with an appended token are bit-identical."""
    lens = [16384, 9000, 64 * 17 + 5, 700]
    b = inputs.make_batch(lens, num_q_heads=32, num_kv_heads=8, seed=89, slack=70)
    kn, vn = inputs.random_kv_rows(len(lens), 8, 128, seed=90, device=DEV)
    g = b.to(DEV)
    p = nosa.params(32, 8, topk=32, kv_int8=True)
    cap = b.capacity.numpy()
    need = [(int(c) + 63) // 64 for c in cap]
    num_pages = sum(need) + 5
    perm = np.random.default_rng(91).permutation(num_pages)
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
    kp_bf = torch.zeros(num_pages * 64, 8, 128, dtype=torch.bfloat16, device=DEV)
    vp_bf = torch.zeros_like(kp_bf)
    kp_bf[dst] = g.k_cache[src]
    vp_bf[dst] = g.v_cache[src]
    kq, vq = _quantized(nosa, p, g)
    kp, vp = nosa.Int8KvCache.from_bf16(p, kp_bf), nosa.Int8KvCache.from_bf16(p, vp_bf)
    table_d = torch.from_numpy(table).to(DEV)
    st_c = nosa.DecodeState(p, b.batch, max(lens) + 1)
    st_p = nosa.DecodeState(p, b.batch, max(lens) + 1)
    st_c.rebuild_pooled(kq, g.seq_start, g.seq_len)
    nosa.nosa_pool_append_paged(p, kp, None, table_d, g.seq_len, st_p.pooled, len_old=torch.zeros_like(g.seq_len),
                                max_new_keys=st_p.nc_cap, ws=st_p.ws)
    assert torch.equal(st_c.pooled, st_p.pooled)
    g.seq_len += 1
    nosa.nosa_decode_step_device(p, g.q, kq, vq, g.seq_start, g.seq_len, st_c.max_seq_len, st_c.pooled,
                                 st_c.sel_idx, st_c.sel_cnt, st_c.out, st_c.ws, k_new=kn, v_new=vn, lse=st_c.lse)
    nosa.nosa_decode_step_device_paged(p, g.q, kp, vp, table_d, g.seq_len, st_p.max_seq_len, st_p.pooled,
                                       st_p.sel_idx, st_p.sel_cnt, st_p.out, st_p.ws, k_new=kn, v_new=vn,
                                       lse=st_p.lse)
    torch.cuda.synchronize()
    for x, y in ((st_c.out, st_p.out), (st_c.lse, st_p.lse), (st_c.sel_idx, st_p.sel_idx),
                 (st_c.pooled, st_p.pooled)):
        assert torch.equal(x, y)
    for i, L in enumerate(lens):
        row_c = int(b.seq_start[i]) + L
        row_p = int(table[i, L // 64]) * 64 + L % 64
        assert torch.equal(kq.codes[row_c], kp.codes[row_p])
        assert torch.equal(kq.row_scales()[row_c], kp.row_scales()[row_p])
    _status_ok(nosa, st_c.ws)
    _status_ok(nosa, st_p.ws)


def test_int8_type_checks(nosa):
    """A bf16 tensor where an INT8 cache is expected (and the reverse) is
    rejected by the binding before any launch."""
    p8 = nosa.params(16, 2, kv_int8=True)
    p16 = nosa.params(16, 2)
    k = torch.zeros(128, 2, 128, dtype=torch.bfloat16, device=DEV)
    c = nosa.Int8KvCache(128, 2)
    seq = torch.zeros(1, dtype=torch.int64, device=DEV)
    ln = torch.full((1,), 64, dtype=torch.int32, device=DEV)
    pooled = torch.zeros(1, 2, 4, 128, device=DEV)
    with pytest.raises(TypeError):
        nosa.nosa_pool_append(p8, k, None, seq, ln, pooled, len_old=torch.zeros_like(ln), max_new_keys=4)
    with pytest.raises(TypeError):
        nosa.nosa_pool_append(p16, c, None, seq, ln, pooled, len_old=torch.zeros_like(ln), max_new_keys=4)
