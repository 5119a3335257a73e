"""Paged KV caches (64-token pages through a page table): the paged entry
points against the contiguous ones on the same tokens (B200).

The caches are scattered into randomly permuted pages; every result must be
bit-identical to the contiguous path (same arithmetic, same tile order), and
the attention output also within tolerance of the oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from helpers import assert_out_close, oracle_step
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


def paginate(b, extra_pages: int, seed: int):
    """(k_pages, v_pages, page_table) holding b's caches in shuffled 64-token pages."""
    cap = b.capacity.cpu().numpy()
    starts = b.seq_start.cpu().numpy()
    need = [(int(c) + 63) // 64 for c in cap]
    max_pages = max(need)
    num_pages = sum(need) + extra_pages
    rng = np.random.default_rng(seed)
    phys = rng.permutation(num_pages)
    table = np.full((b.batch, max_pages), -1, np.int32)
    k = torch.zeros(num_pages * 64, b.num_kv_heads, 128, dtype=torch.bfloat16, device=b.k_cache.device)
    v = torch.zeros_like(k)
    src_rows, dst_rows = [], []
    n = 0
    for i in range(b.batch):
        for pg in range(need[i]):
            table[i, pg] = phys[n]
            n += 1
            t = np.arange(pg * 64, min(pg * 64 + 64, int(cap[i])))
            src_rows.append(int(starts[i]) + t)
            dst_rows.append(int(table[i, pg]) * 64 + (t - pg * 64))
    src = torch.from_numpy(np.concatenate(src_rows)).to(b.k_cache.device)
    dst = torch.from_numpy(np.concatenate(dst_rows)).to(b.k_cache.device)
    k[dst] = b.k_cache[src]
    v[dst] = b.v_cache[src]
    return k, v, torch.from_numpy(table).to(b.k_cache.device)


def _status_ok(nosa, ws):
    rc, bits = nosa.nosa_read_device_status(ws)
    assert rc == 0 and bits == 0, (rc, hex(bits))


@pytest.mark.parametrize("pooled_bf16", [False, True])
def test_paged_fused_step_equals_contiguous(nosa, pooled_bf16):
    lens = [16384, 9000, 3100, 64 * 17 + 5, 700]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=71, slack=70)
    kn, vn = inputs.random_kv_rows(len(lens), 2, 128, seed=72, device=DEV)
    g = b.to(DEV)
    p = nosa.params(16, 2, topk=64, pooled_bf16=pooled_bf16)
    kp, vp, table = paginate(g, extra_pages=9, seed=73)
    st_c = nosa.DecodeState(p, b.batch, max(lens) + 1)
    st_p = nosa.DecodeState(p, b.batch, max(lens) + 1)
    st_c.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    zeros = torch.zeros_like(g.seq_len)
    nosa.nosa_pool_append_paged(p, kp, None, table, g.seq_len, st_p.pooled, len_old=zeros,
                                max_new_keys=st_p.nc_cap, ws=st_p.ws)
    assert torch.equal(st_c.pooled, st_p.pooled)
    g.seq_len += 1                               # one appended token per sequence
    nosa.nosa_decode_step_device(p, g.q, g.k_cache, g.v_cache, g.seq_start, g.seq_len, st_c.max_seq_len,
                                 st_c.pooled, st_c.sel_idx, st_c.sel_cnt, st_c.out, st_c.ws, k_new=kn, v_new=vn,
                                 lse=st_c.lse)
    nosa.nosa_decode_step_device_paged(p, g.q, kp, vp, table, g.seq_len, st_p.max_seq_len, st_p.pooled,
                                       st_p.sel_idx, st_p.sel_cnt, st_p.out, st_p.ws, k_new=kn, v_new=vn,
                                       lse=st_p.lse)
    torch.cuda.synchronize()
    for x, y in ((st_c.out, st_p.out), (st_c.lse, st_p.lse), (st_c.sel_idx, st_p.sel_idx),
                 (st_c.sel_cnt, st_p.sel_cnt), (st_c.pooled, st_p.pooled)):
        assert torch.equal(x, y)
    # the appended rows went to the right physical rows
    tab = table.cpu().numpy()
    for i, L in enumerate(lens):
        row = int(tab[i, L // 64]) * 64 + L % 64
        assert torch.equal(kp[row], kn[i]) and torch.equal(vp[row], vn[i])
    _status_ok(nosa, st_c.ws)
    _status_ok(nosa, st_p.ws)


def test_paged_sparse_decode_matches_contiguous_and_oracle(nosa):
    lens = [8192, 5000, 2049, 64 * 16 + 1]
    b = inputs.make_batch(lens, num_q_heads=32, num_kv_heads=8, seed=74)
    ref = oracle_step(b, 32)
    g = b.to(DEV)
    p = nosa.params(32, 8, topk=32)
    kp, vp, table = paginate(g, extra_pages=3, seed=75)
    sel = torch.from_numpy(ref["sel_idx"]).to(DEV)
    cnt = torch.from_numpy(ref["sel_cnt"]).to(DEV)
    ws = nosa.workspace(p, b.batch, max(lens))
    out_c = torch.empty(b.batch, 32, 128, dtype=torch.bfloat16, device=DEV)
    out_p = torch.empty_like(out_c)
    lse_c = torch.empty(b.batch, 32, device=DEV)
    lse_p = torch.empty_like(lse_c)
    nosa.nosa_sparse_decode(p, g.q, g.k_cache, g.v_cache, g.seq_start, g.seq_len, max(lens), sel, cnt, out_c, ws,
                            lse=lse_c)
    nosa.nosa_sparse_decode_paged(p, g.q, kp, vp, table, g.seq_len, max(lens), sel, cnt, out_p, ws, lse=lse_p)
    torch.cuda.synchronize()
    assert torch.equal(out_c, out_p) and torch.equal(lse_c, lse_p)
    assert_out_close(out_p.float().cpu().numpy(), ref["out"])
    np.testing.assert_allclose(lse_p.cpu().numpy(), ref["lse"], atol=1e-3, rtol=0)
    _status_ok(nosa, ws)


def test_paged_bad_page_index_is_reported(nosa):
    lens = [3000, 2000]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=76)
    g = b.to(DEV)
    p = nosa.params(16, 2, topk=8)
    kp, vp, table = paginate(g, extra_pages=0, seed=77)
    table[1, 20] = kp.shape[0] // 64 + 5         # a local block's page, past the pool
    st = nosa.DecodeState(p, b.batch, max(lens))
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    nosa.nosa_block_select(p, g.q, st.pooled, g.seq_len, max(lens), st.sel_idx, st.sel_cnt, st.ws)
    nosa.nosa_sparse_decode_paged(p, g.q, kp, vp, table, g.seq_len, max(lens), st.sel_idx, st.sel_cnt, st.out,
                                  st.ws)
    rc, bits = nosa.nosa_read_device_status(st.ws)
    assert rc == nosa.NOSA_ERR_DEVICE_CHECK and bits & nosa.NOSA_DEV_BAD_INDEX
    assert torch.isfinite(st.out.float()).all()
