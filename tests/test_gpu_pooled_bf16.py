"""bf16 pooled keys (nosa_params.pooled_bf16): GPU <-> oracle parity (B200).

The pooled mean is rounded to bfloat16 (nearest, ties to even); the GPU sums
in fp32, the oracle in fp64, so a pooled key may differ by one bf16 ulp where
the fp32 and the exact mean round differently.  Scoring is checked on the
oracle's own bf16 pooled keys (exact bf16 products, fp32 accumulation), the
selection bit-exact on separated inputs, the whole step within the usual
attention tolerances."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_out_close, assert_scores_close, assert_valid_topk, oracle_step
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


def _state(nosa, b, topk, max_seq_len=None):
    p = nosa.params(b.num_q_heads, b.num_kv_heads, topk=topk, pooled_bf16=True)
    return p, nosa.DecodeState(p, b.batch, max_seq_len or b.max_seq_len)


def _status_ok(nosa, ws):
    rc, bits = nosa.nosa_read_device_status(ws)
    assert rc == 0 and bits == 0, (rc, hex(bits))


def _bf16_ulp(x):
    a = np.maximum(np.abs(x.astype(np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def test_pool_bf16_matches_oracle(nosa):
    lens = [16384, 5000, 33, 31, 700]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=61)
    g = b.to(DEV)
    p, st = _state(nosa, b, 64)
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    assert st.pooled.dtype == torch.bfloat16
    got = st.pooled.float().cpu().numpy()
    ref = oracle.pool(inputs.bf16_bits(b.k_cache), b.seq_start.numpy(), b.seq_len.numpy(), st.nc_cap, bf16=True)
    for i, L in enumerate(lens):
        nc = oracle.n_windows(L)
        if nc == 0:
            continue
        d = np.abs(got[i, :, :nc] - ref[i, :, :nc])
        assert (d <= _bf16_ulp(ref[i, :, :nc]) * 1.0001).all()
        assert (d == 0).mean() > 0.99
    _status_ok(nosa, st.ws)


def test_pool_bf16_incremental_equals_rebuild(nosa):
    lens = [4096 + 40]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=62, slack=64).to(DEV)
    p, st = _state(nosa, b, 64, max_seq_len=4096 + 80)
    st.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
    for step in range(40):   # append 40 tokens one at a time (crosses two window boundaries)
        kn, vn = inputs.random_kv_rows(1, 2, 128, seed=700 + step, device=DEV)
        b.seq_len += 1
        nosa.nosa_pool_append(p, b.k_cache, b.v_cache, b.seq_start, b.seq_len, st.pooled, max_new_keys=1,
                              k_new=kn, v_new=vn, ws=st.ws)
    inc = st.pooled.clone()
    st.pooled.zero_()
    st.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
    assert torch.equal(inc, st.pooled)
    _status_ok(nosa, st.ws)


@pytest.mark.parametrize("hq,hkv", [(2, 2), (8, 2), (16, 2), (32, 2)])
def test_scores_on_oracle_bf16_pooled_keys(nosa, hq, hkv):
    """Scoring alone: the oracle's bf16 pooled keys are uploaded, so the GPU
    sees exactly the oracle's inputs (exact products, fp32 accumulation)."""
    lens = [9000, 64 * 16 + 64 * 20 + 5, 2100]
    b = inputs.make_batch(lens, num_q_heads=hq, num_kv_heads=hkv, seed=63 + hq)
    ref = oracle_step(b, 64, pooled_bf16=True)
    g = b.to(DEV)
    p, st = _state(nosa, b, 64)
    st.pooled.copy_(torch.from_numpy(ref["pooled"]).to(torch.bfloat16))
    comp = torch.full((b.batch, hq, st.nc_cap), float("nan"), device=DEV)
    bsc = torch.full((b.batch, hkv, nosa.n_blocks(max(lens))), float("nan"), device=DEV)
    nosa.nosa_block_select(p, g.q, st.pooled, g.seq_len, max(lens), st.sel_idx, st.sel_cnt, st.ws,
                           comp_scores_out=comp, block_scores_out=bsc)
    got_c, got_S = comp.cpu().numpy(), bsc.cpu().numpy()
    for i, L in enumerate(lens):
        nc, ncand = oracle.n_windows(L), oracle.n_candidates(L)
        np.testing.assert_allclose(got_c[i, :, :nc], ref["comp_scores"][i, :, :nc], rtol=1e-5,
                                   atol=1e-5 * np.abs(ref["comp_scores"][i, :, :nc]).max())
        assert_scores_close(got_S[i, :, :ncand], ref["block_scores"][i, :, :ncand])
        for h in range(hkv):
            scale = np.max(np.abs(ref["block_scores"][i, h, :ncand])) if ncand else 1.0
            assert_valid_topk(st.sel_idx.cpu().numpy()[i, h], st.sel_cnt.cpu().numpy()[i, h],
                              ref["block_scores"][i, h], ncand, 64, 1e-5 * scale)
    _status_ok(nosa, st.ws)


def test_select_planted_bf16(nosa):
    b = inputs.make_batch(8192, batch=1, num_q_heads=16, num_kv_heads=2, seed=1)
    inputs.plant_blocks(b, seed=101)
    ref = oracle_step(b, 48, pooled_bf16=True)
    g = b.to(DEV)
    p, st = _state(nosa, b, 48)
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    nosa.nosa_block_select(p, g.q, st.pooled, g.seq_len, 8192, st.sel_idx, st.sel_cnt, st.ws)
    np.testing.assert_array_equal(st.sel_idx.cpu().numpy(), ref["sel_idx"])
    np.testing.assert_array_equal(st.sel_cnt.cpu().numpy(), ref["sel_cnt"])
    _status_ok(nosa, st.ws)


def test_full_step_bf16_matches_oracle(nosa):
    lens = [16384, 12000, 3000, 1100, 64 * 17 + 9, 40]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=64)
    ref = oracle_step(b, 64, pooled_bf16=True)
    g = b.to(DEV)
    p, st = _state(nosa, b, 64)
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    st.step(g.q, g.k_cache, g.v_cache, g.seq_start, g.seq_len, append=False, with_lse=True)
    sel, cnt = st.sel_idx.cpu().numpy(), st.sel_cnt.cpu().numpy()
    for i, L in enumerate(lens):
        nc = oracle.n_candidates(L)
        for h in range(2):
            scale = np.max(np.abs(ref["block_scores"][i, h, :nc])) if nc else 1.0
            assert_valid_topk(sel[i, h], cnt[i, h], ref["block_scores"][i, h], nc, 64, 2e-3 * scale)
    same = (sel == ref["sel_idx"]).all(axis=2)
    mask = np.repeat(same, 8, axis=1)
    assert same.mean() > 0.5
    assert_out_close(st.out.float().cpu().numpy()[mask], ref["out"][mask])
    _status_ok(nosa, st.ws)


def test_fused_step_bf16_equals_separate_launches(nosa):
    lens = [16384, 7000, 2500, 16384]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=65, slack=16)
    kn, vn = inputs.random_kv_rows(len(lens), 2, 128, seed=66)
    runs = []
    for fused in (True, False):
        g = b.to(DEV)
        p, st = _state(nosa, b, 64, max_seq_len=max(lens) + 1)
        st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
        g.seq_len += 1
        st.step(g.q, g.k_cache, g.v_cache, g.seq_start, g.seq_len, fused=fused, with_lse=True,
                k_new=kn.to(DEV), v_new=vn.to(DEV))
        torch.cuda.synchronize()
        runs.append((st.out.clone(), st.lse.clone(), st.sel_idx.clone(), st.pooled.clone(), g.k_cache.clone()))
        _status_ok(nosa, st.ws)
    for x, y in zip(runs[0], runs[1]):
        assert torch.equal(x, y)
