"""The fused one-launch decode step equals the three separate launches, bit
for bit, and stays correct over consecutive steps and graph replays (B200)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from helpers import assert_out_close, assert_valid_topk, oracle_step
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


def _pair(nosa, b, topk, max_len, local_blocks=16):
    p = nosa.params(b.num_q_heads, b.num_kv_heads, topk=topk, local_blocks=local_blocks)
    return p, nosa.DecodeState(p, b.batch, max_len), nosa.DecodeState(p, b.batch, max_len)


def _run_both(nosa, b, topk, *, k_new=None, v_new=None, local_blocks=16, steps=1):
    """Separate launches on one copy of the caches, fused on another; compare."""
    ga, gb = b.to(DEV), b.to(DEV)
    max_len = int(b.seq_len.max()) + steps
    p, sa, sb = _pair(nosa, b, topk, max_len, local_blocks)
    lens_a = ga.seq_len.clone()
    sa.rebuild_pooled(ga.k_cache, ga.seq_start, lens_a)
    sb.rebuild_pooled(gb.k_cache, gb.seq_start, lens_a)
    lens = lens_a
    for step in range(steps):
        if k_new is not None:
            lens = lens + 1
        kn = None if k_new is None else k_new[step].to(DEV)
        vn = None if v_new is None else v_new[step].to(DEV)
        sa.step(ga.q, ga.k_cache, ga.v_cache, ga.seq_start, lens, with_lse=True, k_new=kn, v_new=vn)
        sb.step(gb.q, gb.k_cache, gb.v_cache, gb.seq_start, lens, with_lse=True, k_new=kn, v_new=vn,
                fused=True)
        torch.cuda.synchronize()
        assert torch.equal(sa.sel_cnt, sb.sel_cnt)
        assert torch.equal(sa.sel_idx, sb.sel_idx)
        assert torch.equal(sa.out, sb.out), step
        assert torch.equal(sa.lse, sb.lse)
        assert torch.equal(sa.pooled, sb.pooled)
        assert torch.equal(ga.k_cache, gb.k_cache) and torch.equal(ga.v_cache, gb.v_cache)
    for st in (sa, sb):
        rc, bits = nosa.nosa_read_device_status(st.ws)
        assert rc == 0 and bits == 0, hex(bits)
    return sb, gb, lens


@pytest.mark.parametrize("hq,hkv", [(16, 2), (32, 8), (8, 8), (32, 2), (4, 2)])
def test_fused_equals_separate_ragged(nosa, hq, hkv):
    lens = [9000, 3100, 1090, 64 * 40 + 5, 700, 33, 1]
    b = inputs.make_batch(lens, num_q_heads=hq, num_kv_heads=hkv, seed=40 + hq)
    _run_both(nosa, b, 24)


def test_fused_equals_separate_nosa1b_b8_16k(nosa):
    b = inputs.make_batch(16384, batch=8, num_q_heads=16, num_kv_heads=2, seed=2, device=DEV).to("cpu")
    _run_both(nosa, b, 64)


def test_fused_append_steps_equal_separate_and_oracle(nosa):
    """Five consecutive decode steps that each append a token (crossing a pooling
    window boundary), fused vs separate, then the oracle on the final state."""
    lens = [64 * 40 + 12, 5000, 1100]
    steps = 5
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=44, slack=8)
    rows = [inputs.random_kv_rows(3, 2, 128, seed=100 + s) for s in range(steps)]
    kn = [r[0] for r in rows]
    vn = [r[1] for r in rows]
    st, g, final_lens = _run_both(nosa, b, 32, k_new=kn, v_new=vn, steps=steps)
    # host-side cache with the appended rows, for the oracle
    kh, vh = b.k_cache.clone(), b.v_cache.clone()
    for s in range(steps):
        for i, L in enumerate(lens):
            kh[int(b.seq_start[i]) + L + s] = kn[s][i]
            vh[int(b.seq_start[i]) + L + s] = vn[s][i]
    assert torch.equal(kh, g.k_cache.cpu()) and torch.equal(vh, g.v_cache.cpu())
    hb = inputs.DecodeBatch(b.q, kh, vh, b.seq_start, final_lens.cpu(), b.capacity, 16, 2, 128)
    ref = oracle_step(hb, 32)
    sel, cnt = st.sel_idx.cpu().numpy(), st.sel_cnt.cpu().numpy()
    for i in range(3):
        L = int(final_lens[i])
        ncand = max(0, (L + 63) // 64 - 16)
        for h in range(2):
            scale = np.max(np.abs(ref["block_scores"][i, h, :ncand])) if ncand else 1.0
            assert_valid_topk(sel[i, h], cnt[i, h], ref["block_scores"][i, h], ncand, 32, 2e-3 * scale)
    same = np.repeat((sel == ref["sel_idx"]).all(axis=2), 8, axis=1)
    assert same.mean() > 0.5
    assert_out_close(st.out.float().cpu().numpy()[same], ref["out"][same])


def test_fused_small_local_window_falls_back(nosa):
    lens = [3000, 900]
    b = inputs.make_batch(lens, num_q_heads=8, num_kv_heads=2, seed=45)
    _run_both(nosa, b, 8, local_blocks=1)


def test_fused_graph_replay(nosa):
    b = inputs.make_batch([8192, 6000], num_q_heads=16, num_kv_heads=2, seed=46).to(DEV)
    p = nosa.params(16, 2, topk=64)
    st = nosa.DecodeState(p, 2, 8192)
    st.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
    ref = st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len).clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        for _ in range(3):
            st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, fused=True)
    for _ in range(4):
        st.out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(st.out, ref)
    rc, bits = nosa.nosa_read_device_status(st.ws)
    assert rc == 0 and bits == 0, hex(bits)
