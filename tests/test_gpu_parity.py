"""GPU <-> oracle parity of the three kernels, through the C ABI (needs a B200).

Inputs are seeded and synthetic (long_context_decode_nosa_b200.inputs).  The
bar: pooled keys within fp32 summation error; compressed / block scores within
1e-3 relative; block indices bit-exact on separated inputs and when the
oracle's block scores are fed to the selector; attention output within
2e-2 absolute + 1e-2 relative (bf16 out, fp32 accumulate), lse within 1e-3."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from helpers import (assert_out_close, assert_scores_close, assert_valid_topk, oracle_step,
                     sub_batch)
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


def _gpu_state(nosa, b, topk, local_blocks=16, max_seq_len=None):
    p = nosa.params(b.num_q_heads, b.num_kv_heads, topk=topk, local_blocks=local_blocks)
    st = nosa.DecodeState(p, b.batch, max_seq_len or b.max_seq_len)
    return p, st


def _status_ok(nosa, ws):
    rc, bits = nosa.nosa_read_device_status(ws)
    assert rc == 0 and bits == 0, (rc, hex(bits))


# ----------------------------------------------------------------------------- K1 pooling

def test_pool_rebuild_matches_oracle(nosa):
    b = inputs.make_batch([700, 333, 31, 2055, 32, 47], num_q_heads=8, num_kv_heads=2, seed=1)
    g = b.to(DEV)
    p, st = _gpu_state(nosa, b, 8)
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    ref = oracle.pool(inputs.bf16_bits(b.k_cache), b.seq_start.numpy(), b.seq_len.numpy(), st.nc_cap)
    got = st.pooled.cpu().numpy()
    kabs = b.k_cache.abs().double()
    for i in range(b.batch):
        L, s0 = int(b.seq_len[i]), int(b.seq_start[i])
        nc = oracle.n_windows(L)
        if nc == 0:
            continue
        win = kabs[s0:s0 + L].unfold(0, 32, 16).sum(-1).numpy()       # [nc, Hkv, D] sum |k|
        tol = 31 * 2.0 ** -24 * win / 32 + 2.0 ** -24 * np.abs(ref[i, :, :nc].transpose(1, 0, 2))
        err = np.abs(got[i, :, :nc] - ref[i, :, :nc]).transpose(1, 0, 2)
        assert (err <= tol).all(), err.max()
    _status_ok(nosa, st.ws)


def test_pool_incremental_equals_rebuild_bitexact(nosa):
    L0, steps = 500, 70
    b = inputs.make_batch([L0 + steps] * 3, num_q_heads=4, num_kv_heads=2, seed=2)
    g = b.to(DEV)
    p, st = _gpu_state(nosa, b, 8)
    lens = torch.full((3,), L0, dtype=torch.int32, device=DEV)
    nosa.nosa_pool_append(p, g.k_cache, None, g.seq_start, lens, st.pooled,
                          len_old=torch.zeros_like(lens), max_new_keys=st.nc_cap, ws=st.ws)
    for t in range(steps):
        lens += 1
        nosa.nosa_pool_append(p, g.k_cache, None, g.seq_start, lens, st.pooled, max_new_keys=1,
                              ws=st.ws)
    full = torch.zeros_like(st.pooled)
    nosa.nosa_pool_append(p, g.k_cache, None, g.seq_start, lens, full,
                          len_old=torch.zeros_like(lens), max_new_keys=st.nc_cap, ws=st.ws)
    assert torch.equal(st.pooled, full)
    _status_ok(nosa, st.ws)


def test_pool_fused_append_writes_rows_and_pools(nosa):
    L = 64 * 20                       # the appended token L-1 completes window nc(L)-1
    b = inputs.make_batch([L] * 2, num_q_heads=4, num_kv_heads=2, seed=3)
    kn, vn = inputs.random_kv_rows(2, 2, 128, seed=33)
    g = b.to(DEV)
    p, st = _gpu_state(nosa, b, 8)
    lens = g.seq_len.clone()
    st.rebuild_pooled(g.k_cache, g.seq_start, lens - 1)
    nosa.nosa_pool_append(p, g.k_cache, g.v_cache, g.seq_start, lens, st.pooled, max_new_keys=1,
                          k_new=kn.to(DEV), v_new=vn.to(DEV), ws=st.ws)
    for i in range(2):
        row = int(b.seq_start[i]) + L - 1
        assert torch.equal(g.k_cache[row].cpu(), kn[i]) and torch.equal(g.v_cache[row].cpu(), vn[i])
    kh = b.k_cache.clone()
    for i in range(2):
        kh[int(b.seq_start[i]) + L - 1] = kn[i]
    ref = oracle.pool(inputs.bf16_bits(kh), b.seq_start.numpy(), b.seq_len.numpy(), st.nc_cap)
    nc = oracle.n_windows(L)
    np.testing.assert_allclose(st.pooled.cpu().numpy()[:, :, nc - 1], ref[:, :, nc - 1], rtol=2e-6,
                               atol=2e-6)
    _status_ok(nosa, st.ws)


# ----------------------------------------------------------------------------- K2 selection

def test_select_planted_parity_workload(nosa):
    """B=1, 16 q / 2 KV heads, L=8192, top-k 48 of 112, planted blocks: scores
    within 1e-3 and indices bit-exact."""
    b = inputs.make_batch(8192, batch=1, num_q_heads=16, num_kv_heads=2, seed=1)
    inputs.plant_blocks(b, seed=101)
    ref = oracle_step(b, 48)
    g = b.to(DEV)
    p, st = _gpu_state(nosa, b, 48)
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    comp = torch.full((1, 16, st.nc_cap), float("nan"), device=DEV)
    bsc = torch.full((1, 2, nosa.n_blocks(8192)), float("nan"), device=DEV)
    nosa.nosa_block_select(p, g.q, st.pooled, g.seq_len, 8192, st.sel_idx, st.sel_cnt, st.ws,
                           comp_scores_out=comp, block_scores_out=bsc)
    assert_scores_close(comp.cpu().numpy(), ref["comp_scores"])
    assert_scores_close(bsc.cpu().numpy()[:, :, :112], ref["block_scores"][:, :, :112])
    np.testing.assert_array_equal(st.sel_idx.cpu().numpy(), ref["sel_idx"])
    np.testing.assert_array_equal(st.sel_cnt.cpu().numpy(), ref["sel_cnt"])
    _status_ok(nosa, st.ws)


@pytest.mark.parametrize("seed", range(6))
def test_select_only_bitexact_from_oracle_scores(nosa, seed):
    """Selector fed the oracle's fp32 block scores: indices bit-exact, including
    heavy ties, -0.0 and NaN, ragged lengths and every top-k regime."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(1, 64 * 300, size=7).astype(np.int32)
    lens[0] = 64 * 17          # ncand = 1
    lens[1] = 1000             # window only
    nb_cap = oracle.n_blocks(int(lens.max()))
    S = rng.integers(-4, 5, size=(7, 2, nb_cap)).astype(np.float32)     # many ties
    if seed % 2:
        S += rng.standard_normal(S.shape).astype(np.float32)             # few ties
    S[2, 0, :5] = -0.0
    S[2, 1, 3] = np.nan
    for topk in (1, 7, 64, 300):
        idx, cnt = oracle.topk(S, lens, topk)
        p = nosa.params(4, 2, topk=topk)
        ws = nosa.workspace(p, 7, int(lens.max()))
        sel = torch.full((7, 2, topk), -7, dtype=torch.int32, device=DEV)
        sc = torch.zeros(7, 2, dtype=torch.int32, device=DEV)
        nosa.nosa_block_select(p, None, None, torch.from_numpy(lens).to(DEV), int(lens.max()), sel, sc,
                               ws, block_scores_in=torch.from_numpy(S).to(DEV))
        np.testing.assert_array_equal(sel.cpu().numpy(), idx)
        np.testing.assert_array_equal(sc.cpu().numpy(), cnt)
        _status_ok(nosa, ws)


@pytest.mark.parametrize("topk", [1, 64, 96, 700])
def test_select_only_bitexact_many_candidates(nosa, topk):
    """Candidate sets above 1024 (contexts past 66K, up to 128K) take the
    block-wide radix path; 256-1024 the wide warp path; bit-exact either way."""
    rng = np.random.default_rng(topk)
    lens = np.array([131072, 64 * 1100 + 7, 64 * 700, 64 * 250, 5000], np.int32)
    nb_cap = oracle.n_blocks(int(lens.max()))
    S = rng.integers(-6, 7, size=(5, 2, nb_cap)).astype(np.float32)
    S[0, 1] += rng.standard_normal(nb_cap).astype(np.float32)
    idx, cnt = oracle.topk(S, lens, topk)
    p = nosa.params(4, 2, topk=topk)
    ws = nosa.workspace(p, 5, int(lens.max()))
    sel = torch.full((5, 2, topk), -7, dtype=torch.int32, device=DEV)
    sc = torch.zeros(5, 2, dtype=torch.int32, device=DEV)
    nosa.nosa_block_select(p, None, None, torch.from_numpy(lens).to(DEV), int(lens.max()), sel, sc, ws,
                           block_scores_in=torch.from_numpy(S).to(DEV))
    np.testing.assert_array_equal(sel.cpu().numpy(), idx)
    np.testing.assert_array_equal(sc.cpu().numpy(), cnt)
    _status_ok(nosa, ws)


def test_select_unplanted_ragged_valid(nosa):
    """N(0,1) keys, ragged lengths: scores within 1e-3 and the GPU's choice is a
    valid top-k of the oracle's scores (exact wherever the boundary is not a
    near-tie)."""
    lens = [9000, 3100, 1090, 6000, 64 * 16 + 64 * 40]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=4)
    ref = oracle_step(b, 64)
    g = b.to(DEV)
    p, st = _gpu_state(nosa, b, 64)
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    bsc = torch.full((b.batch, 2, nosa.n_blocks(max(lens))), float("nan"), device=DEV)
    nosa.nosa_block_select(p, g.q, st.pooled, g.seq_len, max(lens), st.sel_idx, st.sel_cnt, st.ws,
                           block_scores_out=bsc)
    got_S = bsc.cpu().numpy()
    sel, cnt = st.sel_idx.cpu().numpy(), st.sel_cnt.cpu().numpy()
    for i, L in enumerate(lens):
        nc = oracle.n_candidates(L)
        for h in range(2):
            assert_scores_close(got_S[i, h, :nc], ref["block_scores"][i, h, :nc])
            scale = np.max(np.abs(ref["block_scores"][i, h, :nc])) if nc else 1.0
            assert_valid_topk(sel[i, h], cnt[i, h], ref["block_scores"][i, h], nc, 64, 2e-3 * scale)
    _status_ok(nosa, st.ws)


@pytest.mark.parametrize("L", [5504, 7424, 16384, 65536, 132_000])
def test_select_ties_resolved_to_lowest_index(nosa, L):
    """All keys zero except 10 planted blocks per KV head: every other block
    scores exactly 0, so most of the 64 picks are ties that the lowest block
    index must win -- through the whole scoring path (70 and 100 candidates:
    the sample select ranks tied survivors; 240 and 1008: too many ties for
    its survivor list, so its radix fallback decides; 2047: the radix
    select)."""
    b = inputs.make_batch(L, batch=1, num_q_heads=16, num_kv_heads=2, seed=41)
    b.k_cache.zero_()
    G = 8
    rng = np.random.default_rng(41)
    ncand = oracle.n_candidates(L)
    for h in range(2):
        u = b.q[0, h * G:(h + 1) * G].float().sum(0)
        u = u / u.norm()
        for c in rng.choice(ncand, size=10, replace=False):
            t0 = int(b.seq_start[0]) + 64 * int(c) + 16
            b.k_cache[t0:t0 + 32, h] = (u * float(rng.uniform(1.0, 3.0))).to(torch.bfloat16)
    ref = oracle_step(b, 64)
    g = b.to(DEV)
    p, st = _gpu_state(nosa, b, 64)
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    st.step(g.q, g.k_cache, g.v_cache, g.seq_start, g.seq_len, append=False)
    np.testing.assert_array_equal(st.sel_idx.cpu().numpy(), ref["sel_idx"])
    np.testing.assert_array_equal(st.sel_cnt.cpu().numpy(), ref["sel_cnt"])
    assert_out_close(st.out.float().cpu().numpy(), ref["out"])
    _status_ok(nosa, st.ws)


@pytest.mark.parametrize("hq,hkv,key_dist", [(2, 2, "normal"), (4, 2, "student_t"), (8, 2, "normal"),
                                             (16, 2, "student_t"), (32, 2, "normal"), (32, 8, "student_t")])
def test_select_scores_every_group_size(nosa, hq, hkv, key_dist):
    """Compressed and block scores for group sizes 1..16 (the tensor-core
    scoring tiles the group's heads as the n dimension) on ragged lengths whose
    chunks end mid-tile; heavy-tailed keys exercise the split of each pooled
    value into two TF32 parts."""
    lens = [64 * 16 + 64 * 16 * 3 + 64 * 5 + 9, 2100, 64 * 17, 4097]
    b = inputs.make_batch(lens, num_q_heads=hq, num_kv_heads=hkv, seed=hq + 7 * hkv, key_dist=key_dist)
    ref = oracle_step(b, 64)
    g = b.to(DEV)
    p, st = _gpu_state(nosa, b, 64)
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    comp = torch.full((b.batch, hq, st.nc_cap), float("nan"), device=DEV)
    bsc = torch.full((b.batch, hkv, nosa.n_blocks(max(lens))), float("nan"), device=DEV)
    nosa.nosa_block_select(p, g.q, st.pooled, g.seq_len, max(lens), st.sel_idx, st.sel_cnt, st.ws,
                           comp_scores_out=comp, block_scores_out=bsc)
    got_c, got_S = comp.cpu().numpy(), bsc.cpu().numpy()
    for i, L in enumerate(lens):
        nc, ncand = oracle.n_windows(L), oracle.n_candidates(L)
        assert_scores_close(got_c[i, :, :nc], ref["comp_scores"][i, :, :nc])
        assert_scores_close(got_S[i, :, :ncand], ref["block_scores"][i, :, :ncand])
    _status_ok(nosa, st.ws)


# ----------------------------------------------------------------------------- K3 attention

@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (16, 2), (32, 2), (32, 8)])
def test_decode_matches_oracle_given_oracle_indices(nosa, hq, hkv):
    lens = [5000, 1500, 64 * 30 + 17, 700, 64 * 16 + 64 * 70 + 1]
    b = inputs.make_batch(lens, num_q_heads=hq, num_kv_heads=hkv, seed=5 + hq + hkv)
    ref = oracle_step(b, 24)
    g = b.to(DEV)
    p, st = _gpu_state(nosa, b, 24)
    idx = torch.from_numpy(ref["sel_idx"]).to(DEV)
    cnt = torch.from_numpy(ref["sel_cnt"]).to(DEV)
    nosa.nosa_sparse_decode(p, g.q, g.k_cache, g.v_cache, g.seq_start, g.seq_len, max(lens), idx, cnt,
                            st.out, st.ws, lse=st.lse)
    assert_out_close(st.out.float().cpu().numpy(), ref["out"])
    np.testing.assert_allclose(st.lse.cpu().numpy(), ref["lse"], atol=1e-3, rtol=0)
    # the order of sel_idx does not matter
    rev = ref["sel_idx"].copy()
    for i in range(rev.shape[0]):
        for h in range(rev.shape[1]):
            c = ref["sel_cnt"][i, h]
            rev[i, h, :c] = rev[i, h, :c][::-1]
    out2 = torch.empty_like(st.out)
    nosa.nosa_sparse_decode(p, g.q, g.k_cache, g.v_cache, g.seq_start, g.seq_len, max(lens),
                            torch.from_numpy(rev).to(DEV), cnt, out2, st.ws)
    assert_out_close(out2.float().cpu().numpy(), ref["out"])
    _status_ok(nosa, st.ws)


def test_decode_dense_equivalence(nosa):
    """Budget covering every candidate: the GPU result is dense decode attention."""
    lens = [3000, 64 * 16 + 5, 12, 2049]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=8)
    nb = oracle.n_blocks(max(lens))
    ref = oracle_step(b, nb)
    g = b.to(DEV)
    p, st = _gpu_state(nosa, b, nb)
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    st.step(g.q, g.k_cache, g.v_cache, g.seq_start, g.seq_len, append=False, with_lse=True)
    # dense reference: torch SDPA on the host in fp64
    for i, L in enumerate(lens):
        s0 = int(b.seq_start[i])
        q = b.q[i].double().unsqueeze(1)
        k = b.k_cache[s0:s0 + L].double().permute(1, 0, 2).repeat_interleave(8, 0)
        v = b.v_cache[s0:s0 + L].double().permute(1, 0, 2).repeat_interleave(8, 0)
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v)[:, 0].numpy()
        assert_out_close(st.out[i].float().cpu().numpy(), o)
    assert_out_close(st.out.float().cpu().numpy(), ref["out"])
    np.testing.assert_allclose(st.lse.cpu().numpy(), ref["lse"], atol=1e-3, rtol=0)
    _status_ok(nosa, st.ws)


def test_decode_invariant_to_selection_order(nosa):
    """Attention over a set: permuting each pair's selected indices (which
    moves blocks between the cluster's CTAs and changes the merge order)
    changes the result only by fp32 rounding."""
    lens = [16384, 9000, 5000]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=51).to(DEV)
    p, st = _gpu_state(nosa, b, 64)
    st.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
    st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, append=False, with_lse=True)
    out0, lse0 = st.out.float().clone(), st.lse.clone()
    sel = st.sel_idx.clone()
    rng = np.random.default_rng(51)
    cnt = st.sel_cnt.cpu().numpy()
    for i in range(len(lens)):
        for h in range(2):
            perm = torch.from_numpy(rng.permutation(int(cnt[i, h]))).to(DEV)
            sel[i, h, :cnt[i, h]] = sel[i, h, perm]
    out = torch.empty_like(st.out)
    lse = torch.empty_like(st.lse)
    nosa.nosa_sparse_decode(p, b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, st.max_seq_len, sel,
                            st.sel_cnt, out, st.ws, lse=lse)
    torch.cuda.synchronize()
    np.testing.assert_allclose(out.float().cpu().numpy(), out0.cpu().numpy(), atol=2e-3, rtol=8e-3)
    np.testing.assert_allclose(lse.cpu().numpy(), lse0.cpu().numpy(), atol=1e-5, rtol=1e-6)
    _status_ok(nosa, st.ws)


_PARTITION_SCRIPT = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from long_context_decode_nosa_b200 import inputs, nosa
b = inputs.make_batch([16384, 6000], num_q_heads=16, num_kv_heads=2, seed=52, device="cuda")
p = nosa.params(16, 2, topk=64)
st = nosa.DecodeState(p, b.batch, b.max_seq_len)
st.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, append=False, with_lse=True)
torch.cuda.synchronize()
np.savez(sys.argv[2], out=st.out.float().cpu().numpy(), lse=st.lse.cpu().numpy(),
         sel=st.sel_idx.cpu().numpy())
"""


def test_attention_invariant_to_cluster_partition(nosa, tmp_path):
    """Split-K merge of any partition equals one pass: the same step with one
    CTA per (sequence, KV head) and with clusters of 8 (each CTA a different
    share of the tiles, merged through distributed shared memory) agrees to
    fp32 rounding, and selects the same blocks."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = {}
    for c in (1, 8):
        env = dict(os.environ, NOSA_CLUSTER_SIZE=str(c))
        path = str(tmp_path / f"c{c}.npz")
        subprocess.run([sys.executable, "-c", _PARTITION_SCRIPT, root, path], env=env, check=True, timeout=300)
        res[c] = np.load(path)
    np.testing.assert_array_equal(res[1]["sel"], res[8]["sel"])
    np.testing.assert_allclose(res[1]["lse"], res[8]["lse"], atol=1e-5, rtol=1e-6)
    np.testing.assert_allclose(res[1]["out"], res[8]["out"], atol=2e-3, rtol=8e-3)


_PAIRS_SCRIPT = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from long_context_decode_nosa_b200 import inputs, nosa
b = inputs.make_batch([65536, 40000, 9000, 130], num_q_heads=16, num_kv_heads=2, seed=53, device="cuda")
p = nosa.params(16, 2, topk=64)
st = nosa.DecodeState(p, b.batch, b.max_seq_len)
st.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
bsc = torch.full((b.batch, 2, nosa.n_blocks(b.max_seq_len)), float("nan"), device="cuda")
nosa.nosa_block_select(p, b.q, st.pooled, b.seq_len, b.max_seq_len, st.sel_idx, st.sel_cnt, st.ws,
                       block_scores_out=bsc)
sel0 = st.sel_idx.cpu().numpy()
st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, append=False, with_lse=True)
torch.cuda.synchronize()
rc, bits = nosa.nosa_read_device_status(st.ws)
assert rc == 0, (rc, bits)
np.savez(sys.argv[2], out=st.out.float().cpu().numpy(), lse=st.lse.cpu().numpy(),
         sel=st.sel_idx.cpu().numpy(), sel0=sel0, bsc=bsc.cpu().numpy())
"""


def test_pair_scoring_is_bit_identical(nosa, tmp_path):
    """Scoring two chunks per pass (the deep ring's mode for CTAs with many
    chunks; NOSA_PAIRS forces it on or off, read once per process) performs
    every chunk's arithmetic exactly as the one-chunk pass: block scores,
    selections, outputs and lse are bit-identical, for the fused step and the
    selection launch, over sequences of 64K down to a single candidate."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = {}
    for v in ("0", "1"):
        env = dict(os.environ, NOSA_PAIRS=v)
        path = str(tmp_path / f"p{v}.npz")
        subprocess.run([sys.executable, "-c", _PAIRS_SCRIPT, root, path], env=env, check=True, timeout=300)
        res[v] = np.load(path)
    for key in ("bsc", "sel0", "sel", "lse", "out"):
        np.testing.assert_array_equal(res["0"][key], res["1"][key], err_msg=key)


def test_full_step_edge_lengths(nosa):
    """Lengths at every geometric edge in one ragged batch, whole step."""
    lens = [1, 2, 31, 32, 33, 63, 64, 65, 1023, 1024, 1025, 1088, 1089, 64 * 17 + 63, 2049, 4096]
    b = inputs.make_batch(lens, num_q_heads=8, num_kv_heads=1, seed=9)
    ref = oracle_step(b, 3)
    g = b.to(DEV)
    p, st = _gpu_state(nosa, b, 3)
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    st.step(g.q, g.k_cache, g.v_cache, g.seq_start, g.seq_len, append=False, with_lse=True)
    sel, cnt = st.sel_idx.cpu().numpy(), st.sel_cnt.cpu().numpy()
    np.testing.assert_array_equal(cnt, ref["sel_cnt"])
    for i, L in enumerate(lens):
        nc = oracle.n_candidates(L)
        scale = np.max(np.abs(ref["block_scores"][i, 0, :nc])) if nc else 1.0
        assert_valid_topk(sel[i, 0], cnt[i, 0], ref["block_scores"][i, 0], nc, 3, 2e-3 * scale)
    same = (sel == ref["sel_idx"]).all(axis=(1, 2))
    assert same.sum() >= len(lens) - 2
    assert_out_close(st.out.float().cpu().numpy()[same], ref["out"][same])
    np.testing.assert_allclose(st.lse.cpu().numpy()[same], ref["lse"][same], atol=1e-3, rtol=0)
    _status_ok(nosa, st.ws)


def test_determinism_bitwise(nosa):
    b = inputs.make_batch([16384] * 2, num_q_heads=16, num_kv_heads=2, seed=10).to(DEV)
    p, st = _gpu_state(nosa, b, 64)
    st.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
    o1 = st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, append=False, with_lse=True).clone()
    l1 = st.lse.clone()
    o2 = st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, append=False, with_lse=True)
    assert torch.equal(o1, o2) and torch.equal(l1, st.lse)
    _status_ok(nosa, st.ws)


def test_step_long_context_block_scores_in_workspace(nosa):
    """A 150K-token sequence has 2328 candidates: more than shared memory keeps,
    so its block scores go through the workspace and the selector runs the
    memory-resident top-k.  Planted blocks make the selection exact; one short
    sequence rides along in the same launch."""
    lens = [150_000, 3000]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=31)
    inputs.plant_blocks(b, seed=131)
    ref = oracle_step(b, 64)
    g = b.to(DEV)
    p, st = _gpu_state(nosa, b, 64)
    assert oracle.n_candidates(150_000) > 2048
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    bsc = torch.full((2, 2, nosa.n_blocks(150_000)), float("nan"), device=DEV)
    nosa.nosa_block_select(p, g.q, st.pooled, g.seq_len, 150_000, st.sel_idx, st.sel_cnt, st.ws,
                           block_scores_out=bsc)
    for i, L in enumerate(lens):
        nc = oracle.n_candidates(L)
        assert_scores_close(bsc.cpu().numpy()[i, :, :nc], ref["block_scores"][i, :, :nc])
    np.testing.assert_array_equal(st.sel_idx.cpu().numpy(), ref["sel_idx"])
    np.testing.assert_array_equal(st.sel_cnt.cpu().numpy(), ref["sel_cnt"])
    st.step(g.q, g.k_cache, g.v_cache, g.seq_start, g.seq_len, append=False, with_lse=True)
    np.testing.assert_array_equal(st.sel_idx.cpu().numpy(), ref["sel_idx"])
    assert_out_close(st.out.float().cpu().numpy(), ref["out"])
    np.testing.assert_allclose(st.lse.cpu().numpy(), ref["lse"], atol=1e-3, rtol=0)
    _status_ok(nosa, st.ws)


# ----------------------------------------------------------------------------- full-size workloads

def _compare_sampled(nosa, b_gpu, st, seqs, topk, score_tol=2e-3):
    """Oracle on the sampled sequences; selection valid vs oracle scores,
    output exact-parity wherever the selection equals the oracle's, and the
    attention kernel alone re-run on the oracle's indices everywhere."""
    hb = sub_batch(b_gpu, seqs)
    ref = oracle_step(hb, topk)
    sel = st.sel_idx[seqs].cpu().numpy()
    cnt = st.sel_cnt[seqs].cpu().numpy()
    out = st.out[seqs].float().cpu().numpy()
    for k, i in enumerate(seqs):
        L = int(hb.seq_len[k])
        nc = oracle.n_candidates(L)
        for h in range(hb.num_kv_heads):
            scale = np.max(np.abs(ref["block_scores"][k, h, :nc])) if nc else 1.0
            assert_valid_topk(sel[k, h], cnt[k, h], ref["block_scores"][k, h], nc, topk, score_tol * scale)
    same = (sel == ref["sel_idx"]).all(axis=2)                       # [n, Hkv]
    G = hb.num_q_heads // hb.num_kv_heads
    mask = np.repeat(same, G, axis=1)
    assert same.mean() > 0.5
    assert_out_close(out[mask], ref["out"][mask])
    # attention alone on the oracle's indices, for the sampled sequences
    p = st.p
    ws = nosa.workspace(p, len(seqs), int(hb.seq_len.max()))
    hg = hb.to(DEV)
    o = torch.empty(len(seqs), hb.num_q_heads, 128, dtype=torch.bfloat16, device=DEV)
    nosa.nosa_sparse_decode(p, hg.q, hg.k_cache, hg.v_cache, hg.seq_start, hg.seq_len,
                            int(hb.seq_len.max()), torch.from_numpy(ref["sel_idx"]).to(DEV),
                            torch.from_numpy(ref["sel_cnt"]).to(DEV), o, ws)
    assert_out_close(o.float().cpu().numpy(), ref["out"])


def test_full_size_nosa1b_b8_16k(nosa):
    """NOSA-1B attention shape, batch 8, context 16384, top-k 64 + 16 local blocks,
    in the benchmark's launch configuration; every sequence checked."""
    b = inputs.make_batch(16384, batch=8, num_q_heads=16, num_kv_heads=2, seed=2, device=DEV)
    p, st = _gpu_state(nosa, b, 64)
    st.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
    st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, append=True)
    _status_ok(nosa, st.ws)
    _compare_sampled(nosa, b, st, list(range(8)), 64)


def test_full_size_8b_class_b4_64k(nosa):
    """8B-class shape (32 q / 8 KV heads), batch 4, context 65536, Student-t keys."""
    b = inputs.make_batch(65536, batch=4, num_q_heads=32, num_kv_heads=8, seed=4,
                          key_dist="student_t", device=DEV)
    p, st = _gpu_state(nosa, b, 64)
    st.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
    st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, append=True)
    _status_ok(nosa, st.ws)
    _compare_sampled(nosa, b, st, [0, 3], 64)


def test_full_size_nosa1b_b32_ragged_28_layers(nosa):
    """NOSA-1B shape, batch 32, ragged lengths in [16K, 32K], 28 independent
    layers run back to back; three layers x three sequences sampled."""
    lens = inputs.ragged_lengths(32, 16384, 32768, seed=3)
    layers = []
    for layer in range(28):
        b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=300 + layer, device=DEV)
        p, st = _gpu_state(nosa, b, 64)
        st.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
        layers.append((b, st))
    for b, st in layers:
        st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, append=True)
    torch.cuda.synchronize()
    for layer in (0, 13, 27):
        b, st = layers[layer]
        _status_ok(nosa, st.ws)
        _compare_sampled(nosa, b, st, [0, 17, 31], 64)


# ----------------------------------------------------------------------------- host API, errors

def test_decode_step_host_buffers_equals_device_path(nosa):
    lens = [4000, 2500]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=12, slack=16)
    kn, vn = inputs.random_kv_rows(2, 2, 128, seed=13)
    q = inputs.random_queries(1, 2, 16, 128, seed=14)[0]
    g = b.to(DEV)
    g2 = b.to(DEV)
    p, st = _gpu_state(nosa, b, 64, max_seq_len=max(lens) + 1)
    p2, st2 = _gpu_state(nosa, b, 64, max_seq_len=max(lens) + 1)
    st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
    st2.rebuild_pooled(g2.k_cache, g2.seq_start, g2.seq_len)
    new_len = g.seq_len + 1
    # device path: fused append + select + attend
    nosa.nosa_pool_append(p, g.k_cache, g.v_cache, g.seq_start, new_len, st.pooled, max_new_keys=1,
                          k_new=kn.to(DEV), v_new=vn.to(DEV), ws=st.ws)
    st.step(q.to(DEV), g.k_cache, g.v_cache, g.seq_start, new_len, append=False)
    # host path
    qh, kh, vh = q.pin_memory(), kn.pin_memory(), vn.pin_memory()
    oh = torch.empty(2, 16, 128, dtype=torch.bfloat16).pin_memory()
    nosa.nosa_decode_step(p2, qh, kh, vh, oh, g2.k_cache, g2.v_cache, g2.seq_start, new_len,
                          st2.max_seq_len, st2.pooled, st2.sel_idx, st2.sel_cnt, st2.ws)
    torch.cuda.synchronize()
    assert torch.equal(oh, st.out.cpu())
    assert torch.equal(g.k_cache, g2.k_cache) and torch.equal(st.pooled, st2.pooled)
    # the oracle, on a host cache with the new rows appended on the host
    kh_cache, vh_cache = b.k_cache.clone(), b.v_cache.clone()
    for i, L in enumerate(lens):
        kh_cache[int(b.seq_start[i]) + L] = kn[i]
        vh_cache[int(b.seq_start[i]) + L] = vn[i]
    assert torch.equal(kh_cache, g2.k_cache.cpu()) and torch.equal(vh_cache, g2.v_cache.cpu())
    hb = inputs.DecodeBatch(q, kh_cache, vh_cache, b.seq_start, b.seq_len + 1, b.capacity, 16, 2, 128)
    ref = oracle_step(hb, 64)
    same = np.repeat((st2.sel_idx.cpu().numpy() == ref["sel_idx"]).all(axis=2), 8, axis=1)
    assert same.mean() > 0.5
    assert_out_close(oh.float().numpy()[same], ref["out"][same])
    _status_ok(nosa, st2.ws)


def test_decode_step_packed_equals_three_copies(nosa):
    """nosa_decode_step_packed (q, k_new and v_new back to back in one pinned
    buffer, one copy) gives the same step, bit for bit, as nosa_decode_step
    (three buffers, three copies): output, appended caches, pooled keys and
    selection."""
    lens = [3000, 1700, 5000]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=15, slack=16)
    kn, vn = inputs.random_kv_rows(3, 2, 128, seed=16)
    q = inputs.random_queries(1, 3, 16, 128, seed=17)[0]
    outs = []
    for packed in (False, True):
        g = b.to(DEV)
        p, st = _gpu_state(nosa, b, 64, max_seq_len=max(lens) + 1)
        st.rebuild_pooled(g.k_cache, g.seq_start, g.seq_len)
        oh = torch.empty(3, 16, 128, dtype=torch.bfloat16).pin_memory()
        if packed:
            buf = torch.cat([q.reshape(-1), kn.reshape(-1), vn.reshape(-1)]).pin_memory()
            nosa.nosa_decode_step_packed(p, buf, oh, g.k_cache, g.v_cache, g.seq_start, g.seq_len + 1,
                                         st.max_seq_len, st.pooled, st.sel_idx, st.sel_cnt, st.ws)
        else:
            qh, kh, vh = q.pin_memory(), kn.pin_memory(), vn.pin_memory()
            nosa.nosa_decode_step(p, qh, kh, vh, oh, g.k_cache, g.v_cache, g.seq_start, g.seq_len + 1,
                                  st.max_seq_len, st.pooled, st.sel_idx, st.sel_cnt, st.ws)
        torch.cuda.synchronize()
        _status_ok(nosa, st.ws)
        outs.append((oh.clone(), g.k_cache.cpu(), g.v_cache.cpu(), st.pooled.cpu(), st.sel_idx.cpu(),
                     st.sel_cnt.cpu()))
    for x, y in zip(outs[0], outs[1]):
        assert torch.equal(x, y)


def test_device_checks_report_without_faulting(nosa):
    lens = [3000, 2000]
    b = inputs.make_batch(lens, num_q_heads=4, num_kv_heads=2, seed=15).to(DEV)
    p, st = _gpu_state(nosa, b, 8)
    # an out-of-range selected index: skipped, flagged
    idx = torch.full((2, 2, 8), -1, dtype=torch.int32, device=DEV)
    idx[:, :, 0] = 10_000
    cnt = torch.ones(2, 2, dtype=torch.int32, device=DEV)
    nosa.nosa_sparse_decode(p, b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, 3000, idx, cnt,
                            st.out, st.ws)
    rc, bits = nosa.nosa_read_device_status(st.ws)
    assert rc == nosa.NOSA_ERR_DEVICE_CHECK and bits & nosa.NOSA_DEV_BAD_INDEX
    assert torch.isfinite(st.out.float()).all()
    # a length above max_seq_len: that sequence is skipped, flagged
    nosa.nosa_sparse_decode(p, b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, 2500, st.sel_idx,
                            st.sel_cnt, st.out, st.ws)
    rc, bits = nosa.nosa_read_device_status(st.ws)
    assert rc == nosa.NOSA_ERR_DEVICE_CHECK and bits & nosa.NOSA_DEV_MAX_LEN
    # status is cleared by the read
    rc, bits = nosa.nosa_read_device_status(st.ws)
    assert rc == 0 and bits == 0


def test_bounded_wait_times_out_and_reports(nosa):
    p = nosa.params(16, 2)
    ws = nosa.workspace(p, 1, 1024)
    nosa.nosa_selftest_wait_timeout(ws, max_iters=1000)
    rc, bits = nosa.nosa_read_device_status(ws)
    assert rc == nosa.NOSA_ERR_TIMEOUT and bits & nosa.NOSA_DEV_TIMEOUT
    # the context is still usable
    x = torch.ones(4, device=DEV)
    assert float(x.sum()) == 4.0


def test_cuda_graph_capture_of_a_step(nosa):
    b = inputs.make_batch([8192] * 2, num_q_heads=16, num_kv_heads=2, seed=16).to(DEV)
    p, st = _gpu_state(nosa, b, 64)
    st.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
    ref = st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, append=True).clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        st.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, append=True)
    st.out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(st.out, ref)
    _status_ok(nosa, st.ws)
