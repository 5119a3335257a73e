"""Pins of the CPU oracle against things other than itself (CPU only).

Each test ties one oracle function to a closed form, a literal fixture from
``tests/golden/`` (with its citation), a brute-force enumeration on tiny
inputs, or a library routine (numpy sliding-window means, torch's
scaled_dot_product_attention in fp64)."""
from __future__ import annotations

import itertools
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from long_context_decode_nosa_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _bits(t):
    return inputs.bf16_bits(t)


# --------------------------------------------------------------------------- geometry

def test_geometry_golden(oracle_mod):
    """Window / block / candidate counts against the literal table derived from
    the pages' parameters (golden/geometry.txt)."""
    for L, nc, nb, ncand, _local in (map(int, r) for r in _rows("geometry.txt")):
        assert oracle_mod.n_windows(L) == nc, L
        assert oracle_mod.n_blocks(L) == nb, L
        assert oracle_mod.n_candidates(L) == ncand, L


@pytest.mark.parametrize("L", [1, 31, 32, 47, 1024, 1025, 1088, 1089])
def test_geometry_local_window_tokens(oracle_mod, L):
    """With nothing selected, attention covers exactly the last local_tokens(L)
    tokens of golden/geometry.txt (checked through attention weights: V is the
    one-hot token index, so the output is the attention distribution)."""
    table = {int(r[0]): int(r[4]) for r in _rows("geometry.txt")}
    local = table[L]
    hkv, d = 1, 128
    b = inputs.make_batch(L, batch=1, num_q_heads=1, num_kv_heads=hkv, seed=5)
    # zero query -> uniform weights over the attended set
    q = torch.zeros(1, 1, d, dtype=torch.bfloat16)
    idx = np.full((1, 1, 4), -1, np.int32)
    cnt = np.zeros((1, 1), np.int32)
    out, lse = oracle_mod.sparse_attention(_bits(q), _bits(b.k_cache), _bits(b.v_cache),
                                           b.seq_start.numpy(), b.seq_len.numpy(), idx, cnt)
    vf = b.v_cache.double()[:, 0, :].numpy()
    np.testing.assert_allclose(out[0, 0], vf[L - local:L].mean(0), rtol=1e-12, atol=1e-12)
    assert abs(lse[0, 0] - math.log(local)) < 1e-12


# --------------------------------------------------------------------------- pooling

def test_pool_is_window_mean(oracle_mod):
    """Pooled key j = mean of keys [16j, 16j+32) (closed form via numpy's
    sliding_window_view).  fp64 sums of 32 bf16 values of these magnitudes are
    exact, so both sides round the same real number to fp32: bit-exact."""
    b = inputs.make_batch([700, 333, 31], num_kv_heads=2, num_q_heads=4, seed=11)
    nc_cap = oracle_mod.n_windows(700)
    pooled = oracle_mod.pool(_bits(b.k_cache), b.seq_start.numpy(), b.seq_len.numpy(), nc_cap)
    kf = b.k_cache.double().numpy()
    for i in range(3):
        L, s0 = int(b.seq_len[i]), int(b.seq_start[i])
        nc = oracle_mod.n_windows(L)
        if nc:
            win = np.lib.stride_tricks.sliding_window_view(kf[s0:s0 + L], 32, axis=0)[::16]
            ref = win.mean(-1).astype(np.float32)  # [nc, Hkv, D]
            assert ref.shape[0] == nc
            np.testing.assert_array_equal(pooled[i, :, :nc], ref.transpose(1, 0, 2))
        assert not pooled[i, :, nc:].any()


def test_pool_incremental_equals_rebuild(oracle_mod):
    """Appending tokens one at a time gives the same pooled cache as one rebuild,
    and windows outside [nc(len_old), nc(len_new)) are left alone."""
    L = 300
    b = inputs.make_batch(L, batch=2, num_kv_heads=2, num_q_heads=2, seed=3)
    nc_cap = oracle_mod.n_windows(L)
    full = oracle_mod.pool(_bits(b.k_cache), b.seq_start.numpy(), b.seq_len.numpy(), nc_cap)
    inc = np.full_like(full, 7.0)
    inc[:] = 0
    for t in range(1, L + 1):
        lo = np.full(2, t - 1, np.int32)
        hi = np.full(2, t, np.int32)
        inc = oracle_mod.pool(_bits(b.k_cache), b.seq_start.numpy(), hi, nc_cap, len_old=lo,
                              pooled=inc)
    np.testing.assert_array_equal(inc, full)
    sentinel = np.full_like(full, 7.0)
    out = oracle_mod.pool(_bits(b.k_cache), b.seq_start.numpy(), np.full(2, 100, np.int32),
                          nc_cap, len_old=np.full(2, 50, np.int32), pooled=sentinel)
    lo, hi = oracle_mod.n_windows(50), oracle_mod.n_windows(100)
    np.testing.assert_array_equal(out[:, :, lo:hi], full[:, :, lo:hi])
    assert (out[:, :, :lo] == 7.0).all() and (out[:, :, hi:] == 7.0).all()


# --------------------------------------------------------------------------- scores

def test_comp_scores_equal_mean_of_token_scores(oracle_mod):
    """Linearity: scale * q . mean(k_t) equals the mean over the window of the
    per-token scores scale * q . k_t (so pooling keys and pooling raw scores
    agree).  Token scores via numpy einsum in fp64."""
    b = inputs.make_batch([520, 97], num_q_heads=8, num_kv_heads=2, seed=21)
    nc_cap = oracle_mod.n_windows(520)
    pooled = oracle_mod.pool(_bits(b.k_cache), b.seq_start.numpy(), b.seq_len.numpy(), nc_cap)
    s = oracle_mod.comp_scores(_bits(b.q), pooled, b.seq_len.numpy(), num_kv_heads=2)
    qf, kf = b.q.double().numpy(), b.k_cache.double().numpy()
    scale = 1 / math.sqrt(128)
    for i in range(2):
        L, s0 = int(b.seq_len[i]), int(b.seq_start[i])
        nc = oracle_mod.n_windows(L)
        tok = scale * np.einsum("hd,thd->ht", qf[i], np.repeat(kf[s0:s0 + L], 4, axis=1))
        win = np.lib.stride_tricks.sliding_window_view(tok, 32, axis=1)[:, ::16].mean(-1)
        np.testing.assert_allclose(s[i, :, :nc], win, rtol=2e-6, atol=2e-6)
        assert np.isneginf(s[i, :, nc:]).all()


def test_comp_scores_gqa_mapping(oracle_mod):
    """Query head h reads KV head h // G: a one-hot query along dim c returns
    scale * pooled[g][:, c] for its own group only."""
    rng = np.random.default_rng(0)
    B, hq, hkv, d, nc = 1, 4, 2, 128, 5
    pooled = rng.standard_normal((B, hkv, nc, d)).astype(np.float32)
    q = torch.zeros(B, hq, d, dtype=torch.bfloat16)
    for h in range(hq):
        q[0, h, 10 + h] = 1.0
    L = np.array([32 + 16 * (nc - 1)], np.int32)
    s = oracle_mod.comp_scores(_bits(q), pooled, L, num_kv_heads=hkv, scale=1.0)
    for h in range(hq):
        np.testing.assert_array_equal(s[0, h], pooled[0, h // 2, :, 10 + h])


# --------------------------------------------------------------------------- block scores

def test_block_overlap_golden(oracle_mod):
    """A one-hot compressed score at window j lights exactly the blocks of
    golden/block_overlap.txt."""
    L = 64 * 40
    nc = oracle_mod.n_windows(L)
    nb = oracle_mod.n_blocks(L)
    for row in _rows("block_overlap.txt"):
        j = int(row[0])
        want = sorted(int(x) for x in row[3].split(","))
        s = np.zeros((1, 1, nc), np.float32)
        s[0, 0, j] = 1.0
        S = oracle_mod.block_scores(s, np.array([L], np.int32), nb, num_kv_heads=1)
        lit = sorted(np.nonzero(S[0, 0, :nb - 16] == 1.0)[0].tolist())
        assert lit == want, (j, lit, want)


def test_block_scores_max_then_sum_over_group(oracle_mod):
    """Literal values: max over a block's windows per head, summed over the
    heads of the GQA group; -inf outside the candidates."""
    L = 64 * 20  # 20 blocks, 4 candidates
    nc = oracle_mod.n_windows(L)
    s = np.full((1, 4, nc), -1.0, np.float32)   # heads 0,1 -> KV head 0; 2,3 -> KV head 1
    s[0, 0, 4] = 1.0    # block 1
    s[0, 0, 5] = 3.0    # block 1
    s[0, 1, 7] = 2.0    # blocks 1, 2
    s[0, 2, 0] = 5.0    # block 0
    s[0, 3, 15] = 4.0   # blocks 3, 4 (4 is local)
    S = oracle_mod.block_scores(s, np.array([L], np.int32), 20, num_kv_heads=2)
    np.testing.assert_array_equal(S[0, 0, :4], np.array([-2.0, 5.0, 1.0, -2.0], np.float32))
    np.testing.assert_array_equal(S[0, 1, :4], np.array([4.0, -2.0, -2.0, 3.0], np.float32))
    assert np.isneginf(S[0, :, 4:]).all()


# --------------------------------------------------------------------------- top-k

def _brute_topk(scores, k):
    """The unique size-k subset X with: for x in X, y not in X, x ranks above y
    (higher score, or equal score and lower index); NaN ranks as -inf and
    -0.0 equals +0.0."""
    n = len(scores)
    val = [(-math.inf if math.isnan(v) else (0.0 if v == 0 else v)) for v in scores]

    def above(x, y):
        return val[x] > val[y] or (val[x] == val[y] and x < y)

    found = [X for X in itertools.combinations(range(n), k)
             if all(above(x, y) for x in X for y in set(range(n)) - set(X))]
    assert len(found) == 1
    return list(found[0])


@pytest.mark.parametrize("seed", range(40))
def test_topk_brute_force(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    ncand = int(rng.integers(0, 13))
    L = 64 * (ncand + 16)
    # few distinct values -> many ties; sprinkle -0.0, +0.0 and NaN
    S = rng.integers(-3, 4, size=(1, 1, ncand + 16)).astype(np.float32)
    if ncand and seed % 3 == 0:
        S[0, 0, rng.integers(0, ncand)] = -0.0
        S[0, 0, rng.integers(0, ncand)] = np.nan
    for k in sorted({1, ncand // 2, ncand - 1, ncand, ncand + 3} - {0, -1}):
        idx, cnt = oracle_mod.topk(S, np.array([L], np.int32), k)
        kk = min(k, ncand)
        assert cnt[0, 0] == kk
        want = _brute_topk(S[0, 0, :ncand].tolist(), kk)
        assert idx[0, 0, :kk].tolist() == want
        assert (idx[0, 0, kk:] == -1).all()


def test_topk_ties_go_to_lowest_index(oracle_mod):
    S = np.zeros((1, 1, 26), np.float32)  # 10 candidates, all tied
    idx, cnt = oracle_mod.topk(S, np.array([64 * 26], np.int32), 4)
    assert idx[0, 0].tolist() == [0, 1, 2, 3] and cnt[0, 0] == 4


# --------------------------------------------------------------------------- attention

def _sdpa_reference(b, mask_tokens, i, scale=None):
    """torch fp64 scaled_dot_product_attention of sequence i over a token mask."""
    G = b.num_q_heads // b.num_kv_heads
    L, s0 = int(b.seq_len[i]), int(b.seq_start[i])
    q = b.q[i].double().unsqueeze(1)                           # [Hq, 1, D]
    k = b.k_cache[s0:s0 + L].double().permute(1, 0, 2).repeat_interleave(G, 0)
    v = b.v_cache[s0:s0 + L].double().permute(1, 0, 2).repeat_interleave(G, 0)
    m = torch.as_tensor(mask_tokens)                           # [Hkv, L] bool
    m = m.repeat_interleave(G, 0).unsqueeze(1)                 # [Hq, 1, L]
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)
    logits = (q @ k.transpose(-1, -2)) * (scale if scale else 1 / math.sqrt(b.head_dim))
    lse = torch.logsumexp(logits.masked_fill(~m, -math.inf), dim=-1)
    return o[:, 0].numpy(), lse[:, 0].numpy()


def test_dense_equivalence_when_budget_covers_all(oracle_mod):
    """topk >= number of candidates: sparse attention == dense causal decode
    attention over [0, L) (library SDPA in fp64)."""
    lens = [1500, 2300, 700, 64 * 17 + 5]
    b = inputs.make_batch(lens, num_q_heads=8, num_kv_heads=2, seed=7)
    nb_max = oracle_mod.n_blocks(max(lens))
    idx = np.full((4, 2, nb_max), -1, np.int32)
    cnt = np.zeros((4, 2), np.int32)
    for i, L in enumerate(lens):
        nc = oracle_mod.n_candidates(L)
        idx[i, :, :nc] = np.arange(nc)
        cnt[i, :] = nc
    out, lse = oracle_mod.sparse_attention(_bits(b.q), _bits(b.k_cache), _bits(b.v_cache),
                                           b.seq_start.numpy(), b.seq_len.numpy(), idx, cnt)
    for i, L in enumerate(lens):
        o_ref, l_ref = _sdpa_reference(b, np.ones((2, L), bool), i)
        np.testing.assert_allclose(out[i], o_ref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse[i], l_ref, rtol=1e-12, atol=1e-12)


def test_sparse_set_matches_masked_sdpa(oracle_mod):
    """A hand-picked selection: output equals masked SDPA over the literal token
    set (selected blocks + block-aligned local window)."""
    L = 64 * 30 + 17                      # nb = 31, ncand = 15, local = [960, L)
    b = inputs.make_batch(L, batch=1, num_q_heads=4, num_kv_heads=2, seed=9)
    sel = {0: [0, 3, 14], 1: [2, 7]}
    idx = np.full((1, 2, 3), -1, np.int32)
    cnt = np.zeros((1, 2), np.int32)
    mask = np.zeros((2, L), bool)
    for g, blocks in sel.items():
        idx[0, g, :len(blocks)] = blocks
        cnt[0, g] = len(blocks)
        for blk in blocks:
            mask[g, 64 * blk:64 * blk + 64] = True
        mask[g, 960:] = True
    out, lse = oracle_mod.sparse_attention(_bits(b.q), _bits(b.k_cache), _bits(b.v_cache),
                                           b.seq_start.numpy(), b.seq_len.numpy(), idx, cnt,
                                           scale=0.3)
    o_ref, l_ref = _sdpa_reference(b, mask, 0, scale=0.3)
    np.testing.assert_allclose(out[0], o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse[0], l_ref, rtol=1e-12, atol=1e-12)


def test_attention_invariant_to_selection_order(oracle_mod):
    L = 64 * 40
    b = inputs.make_batch(L, batch=1, num_q_heads=2, num_kv_heads=1, seed=13)
    idx = np.array([[[1, 5, 9, 20]]], np.int32)
    cnt = np.array([[4]], np.int32)
    a = oracle_mod.sparse_attention(_bits(b.q), _bits(b.k_cache), _bits(b.v_cache),
                                    b.seq_start.numpy(), b.seq_len.numpy(), idx, cnt)
    c = oracle_mod.sparse_attention(_bits(b.q), _bits(b.k_cache), _bits(b.v_cache),
                                    b.seq_start.numpy(), b.seq_len.numpy(),
                                    idx[:, :, ::-1].copy(), cnt)
    np.testing.assert_allclose(a[0], c[0], rtol=1e-13, atol=1e-15)


def test_attention_rejects_out_of_range_index(oracle_mod):
    L = 64 * 20
    b = inputs.make_batch(L, batch=1, num_q_heads=2, num_kv_heads=1, seed=1)
    idx = np.array([[[4]]], np.int32)     # ncand = 4 -> index 4 is local, not a candidate
    with pytest.raises(ValueError):
        oracle_mod.sparse_attention(_bits(b.q), _bits(b.k_cache), _bits(b.v_cache),
                                    b.seq_start.numpy(), b.seq_len.numpy(), idx,
                                    np.array([[1]], np.int32))


# --------------------------------------------------------------------------- whole step

def test_planted_blocks_are_selected_with_a_clear_gap(oracle_mod):
    """Parity workload shape (B=1, 16/2 heads, L=8192, top-k 48 of 112): every
    planted block is selected and the top-k boundary gap is far above fp32
    score rounding."""
    b = inputs.make_batch(8192, batch=1, num_q_heads=16, num_kv_heads=2, seed=1)
    planted = inputs.plant_blocks(b, seed=101)
    nc_cap = oracle_mod.n_windows(8192)
    pooled = oracle_mod.pool(_bits(b.k_cache), b.seq_start.numpy(), b.seq_len.numpy(), nc_cap)
    r = oracle_mod.decode_step(_bits(b.q), _bits(b.k_cache), _bits(b.v_cache),
                               b.seq_start.numpy(), b.seq_len.numpy(), pooled, 48)
    for g in range(2):
        sel = set(r["sel_idx"][0, g].tolist())
        assert set(planted[0, g].tolist()) <= sel
        S = np.sort(r["block_scores"][0, g, :112])[::-1]
        gap = S[47] - S[48]
        assert gap > 1e-3 * max(1.0, abs(S[47])), gap


# ----------------------------------------------------------------------------- bf16 pooled keys

def test_round_bf16_matches_torch_conversion(oracle_mod):
    """The oracle's own round-to-nearest-even against torch's fp32 -> bfloat16
    conversion: random values over many magnitudes, exact halfway cases with
    an even and an odd kept bit, subnormals, the largest finite values and
    the infinities."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-40, 40, 20000))).astype(np.float32)
    kept = rng.integers(0, 1 << 16, 4000, dtype=np.uint32) << 16
    kept = kept[(kept & 0x7F800000) != 0x7F800000]                   # no NaN / infinity patterns
    halves = (kept | 0x8000).view(np.float32)                       # exactly halfway
    sub = (rng.integers(1, 1 << 23, 2000, dtype=np.uint32)).view(np.float32)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, -3.3895314e38, 3.4028235e38,
                        1.0, 1.00390625, 1.005859375], np.float32)
    allx = np.concatenate([x, halves, sub, special])
    want = torch.from_numpy(allx).to(torch.bfloat16).float().numpy()
    got = oracle_mod.round_bf16(allx)
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
    nan = oracle_mod.round_bf16(np.array([np.nan], np.float32))
    assert np.isnan(nan).all()


def test_pool_bf16_within_half_ulp_of_window_mean(oracle_mod):
    """bf16 pooled keys are bfloat16 values within half a bf16 ulp (plus the
    fp32 rounding of the mean) of the exact fp64 mean of the window's keys."""
    b = inputs.make_batch([300, 77], num_q_heads=4, num_kv_heads=2, seed=6)
    kb = inputs.bf16_bits(b.k_cache)
    lens = b.seq_len.numpy()
    nc_cap = oracle_mod.n_windows(300)
    pb = oracle_mod.pool(kb, b.seq_start.numpy(), lens, nc_cap, bf16=True)
    assert np.array_equal(pb.view(np.uint32) & 0xFFFF, np.zeros_like(pb.view(np.uint32)))
    k = b.k_cache.double().numpy()
    for i, L in enumerate(lens):
        s0 = int(b.seq_start[i])
        for j in range(oracle_mod.n_windows(int(L))):
            exact = k[s0 + 16 * j:s0 + 16 * j + 32].mean(axis=0)       # [Hkv, D]
            ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 1e-30))) - 7)
            err = np.abs(pb[i, :, j] - exact)
            assert (err <= 0.5 * ulp * (1 + 2 ** -20) + 2.0 ** -126).all(), (i, j)


# --------------------------------------------------------------------------- INT8 cache variant

def _pow2_grid_rows(rng, rows, d):
    """Rows k * 2^e (k integer in [-127, 127], one |k| = 127 per row): every
    value has at most 7 significant bits, so it is an exact bfloat16."""
    k = rng.integers(-127, 128, (rows, d))
    k[np.arange(rows), rng.integers(0, d, rows)] = 127 * rng.choice([-1, 1], rows)
    e = rng.integers(-30, 12, rows)
    x = torch.from_numpy(k * np.exp2(e)[:, None]).to(torch.bfloat16)
    assert torch.equal(x.double(), torch.from_numpy(k * np.exp2(e)[:, None]))
    return x, k, e


def test_quantize_int8_reproduces_a_power_of_two_grid(oracle_mod):
    """A row k * 2^e with max |k| = 127 quantizes to scale 2^e and codes k
    exactly (the scale divides out exactly, no rounding is involved)."""
    rng = np.random.default_rng(21)
    x, k, e = _pow2_grid_rows(rng, 300, 128)
    codes, scales = oracle_mod.quantize_int8(_bits(x))
    np.testing.assert_array_equal(scales, np.exp2(e).astype(np.float32))
    np.testing.assert_array_equal(codes, k.astype(np.int8))


def test_quantize_int8_rounds_half_to_even(oracle_mod):
    """Values exactly halfway between two codes go to the even code: 2.5 -> 2,
    3.5 -> 4, 126.5 -> 126, 125.5 -> 126 and the mirrored negatives (half away
    from zero would give 3 and 127)."""
    e = -3
    halves = np.array([0.5, 1.5, 2.5, 3.5, 125.5, 126.5])
    want = np.array([0, 2, 2, 4, 126, 126])
    row = np.concatenate([[127.0], halves, -halves, np.zeros(128 - 13)]) * 2.0 ** e
    x = torch.from_numpy(row[None]).to(torch.bfloat16)
    assert torch.equal(x.double()[0], torch.from_numpy(row))
    codes, scales = oracle_mod.quantize_int8(_bits(x))
    assert scales[0] == np.float32(2.0 ** e)
    np.testing.assert_array_equal(codes[0, 1:7], want)
    np.testing.assert_array_equal(codes[0, 7:13], -want)


def test_quantize_int8_properties_on_random_rows(oracle_mod):
    """On Gaussian rows of many magnitudes, and an all-zero row: the largest
    |code| is 127, codes keep the sign of their value and its order within a
    row, every value lies within half a step (plus the fp32 rounding of x / s)
    of s * code, and the zero row has scale 0 and zero codes."""
    rng = np.random.default_rng(22)
    x = rng.standard_normal((400, 128)) * np.exp(rng.uniform(-20, 20, (400, 1)))
    x[7] = 0.0
    xb = torch.from_numpy(x).to(torch.bfloat16)
    codes, scales = oracle_mod.quantize_int8(_bits(xb))
    xv = xb.double().numpy()
    c = codes.astype(np.int64)
    s = scales.astype(np.float64)
    nz = np.abs(xv).max(1) > 0
    assert (np.abs(c[nz]).max(1) == 127).all()
    assert scales[7] == 0.0 and (codes[7] == 0).all()
    assert ((np.sign(c) == np.sign(xv)) | (c == 0)).all()
    assert (np.abs(xv - s[:, None] * c) <= s[:, None] * (0.5 + 2.0 ** -16)).all()
    order = np.argsort(xv, axis=1, kind="stable")
    assert (np.diff(np.take_along_axis(c, order, 1), axis=1) >= 0).all()
    # the scale is the fp32 quotient of the row's largest magnitude by 127
    amax = np.abs(xv).max(1)
    assert (np.abs(s - amax / 127) <= np.spacing(np.float32(amax / 127)).astype(np.float64)).all()


def _int8_cache(rng, T, hkv, d, pow2_scales):
    codes = rng.integers(-127, 128, (T, hkv, d)).astype(np.int8)
    if pow2_scales:
        scales = np.exp2(rng.integers(-12, 4, (T, hkv))).astype(np.float32)
    else:
        scales = (rng.uniform(0.5, 2.0, (T, hkv)) * np.exp2(rng.integers(-10, 2, (T, hkv)))).astype(np.float32)
    return codes, scales


def _dequant_bf16(codes, scales):
    """s * code as bfloat16 bits (exact when s is a power of two)."""
    v = codes.astype(np.float64) * scales.astype(np.float64)[..., None]
    t = torch.from_numpy(v).to(torch.bfloat16)
    assert torch.equal(t.double(), torch.from_numpy(v))
    return _bits(t)


def test_pool_int8_equals_pool_of_dequantized_keys(oracle_mod):
    """With power-of-two scales every s * code is an exact bfloat16, so pooling
    the INT8 cache must give the bf16 pooling's bits; with general scales the
    pooled key is the fp32 rounding of the window mean of s * code (numpy
    sliding windows in fp64)."""
    rng = np.random.default_rng(23)
    lens = np.array([300, 77, 31], np.int32)
    starts = np.array([0, 300, 377], np.int64)
    nc_cap = oracle_mod.n_windows(300)
    codes, scales = _int8_cache(rng, 408, 2, 128, True)
    got = oracle_mod.pool_int8(codes, scales, starts, lens, nc_cap)
    want = oracle_mod.pool(_dequant_bf16(codes, scales), starts, lens, nc_cap)
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
    codes, scales = _int8_cache(rng, 408, 2, 128, False)
    got = oracle_mod.pool_int8(codes, scales, starts, lens, nc_cap)
    v = codes.astype(np.float64) * scales.astype(np.float64)[..., None]
    for i, L in enumerate(lens):
        nc = oracle_mod.n_windows(int(L))
        if nc == 0:
            continue
        win = np.lib.stride_tricks.sliding_window_view(v[starts[i]:starts[i] + L], 32, axis=0)[::16][:nc]
        mean = win.mean(axis=-1).transpose(1, 0, 2)                     # [Hkv, nc, D]
        np.testing.assert_allclose(got[i, :, :nc], mean, rtol=2.0 ** -23, atol=0)


def test_attention_int8_equals_attention_of_dequantized_cache(oracle_mod):
    """Power-of-two scales: INT8 attention == bf16 attention over the exact
    dequantized cache, bit for bit (same fp64 values, same order).  General
    scales: equal to torch's fp64 SDPA over s * code with the token mask of the
    selection plus the local window."""
    rng = np.random.default_rng(24)
    L = 64 * 30 + 17                                                    # ncand = 15
    b = inputs.make_batch(L, batch=1, num_q_heads=4, num_kv_heads=2, seed=25)
    idx = np.array([[[0, 3, 14], [2, 7, -1]]], np.int32)
    cnt = np.array([[3, 2]], np.int32)
    for pow2 in (True, False):
        kc, ks = _int8_cache(rng, L, 2, 128, pow2)
        vc, vs = _int8_cache(rng, L, 2, 128, pow2)
        out, lse = oracle_mod.sparse_attention_int8(_bits(b.q), kc, ks, vc, vs, b.seq_start.numpy(),
                                                    b.seq_len.numpy(), idx, cnt)
        if pow2:
            o2, l2 = oracle_mod.sparse_attention(_bits(b.q), _dequant_bf16(kc, ks), _dequant_bf16(vc, vs),
                                                 b.seq_start.numpy(), b.seq_len.numpy(), idx, cnt)
            np.testing.assert_array_equal(out, o2)
            np.testing.assert_array_equal(lse, l2)
            continue
        mask = np.zeros((2, L), bool)
        for g in range(2):
            for blk in idx[0, g, :cnt[0, g]]:
                mask[g, 64 * blk:64 * blk + 64] = True
            mask[g, 960:] = True
        kd = torch.from_numpy(kc.astype(np.float64) * ks.astype(np.float64)[..., None])
        vd = torch.from_numpy(vc.astype(np.float64) * vs.astype(np.float64)[..., None])
        q = b.q[0].double().unsqueeze(1)
        k = kd.permute(1, 0, 2).repeat_interleave(2, 0)
        v = vd.permute(1, 0, 2).repeat_interleave(2, 0)
        m = torch.from_numpy(mask).repeat_interleave(2, 0).unsqueeze(1)
        o_ref = F.scaled_dot_product_attention(q, k, v, attn_mask=m)[:, 0].numpy()
        logits = (q @ k.transpose(-1, -2)) / math.sqrt(128)
        l_ref = torch.logsumexp(logits.masked_fill(~m, -math.inf), dim=-1)[:, 0].numpy()
        np.testing.assert_allclose(out[0], o_ref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse[0], l_ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- sparse prefill

def test_sparse_prefill_is_causal_attention_when_budget_covers_all(oracle_mod):
    """With a top-k at least the number of candidates of every prefix, each
    prefill token attends to exactly its whole prefix: the output is causal
    attention (torch fp64 SDPA with a lower-triangular mask over the chunk's
    rows), which pins the per-token length L = position + 1."""
    lens = [2100, 1500]
    b = inputs.make_batch(lens, num_q_heads=4, num_kv_heads=2, seed=31)
    rows = [(1900, 200), (0, 1500)]                      # (first position, rows) per sequence
    q_pos = np.array([r[0] for r in rows], np.int32)
    q_start = np.concatenate([[0], np.cumsum([r[1] for r in rows])]).astype(np.int32)
    total_q = int(q_start[-1])
    gen = torch.Generator().manual_seed(32)
    qf = torch.randn(total_q, 4, 128, generator=gen).to(torch.bfloat16)
    nc_cap = oracle_mod.n_windows(max(lens))
    pooled = oracle_mod.pool(_bits(b.k_cache), b.seq_start.numpy(), b.seq_len.numpy(), nc_cap)
    topk = oracle_mod.n_candidates(max(lens))
    sel, cnt, out, lse = oracle_mod.sparse_prefill(_bits(qf), _bits(b.k_cache), _bits(b.v_cache),
                                                   b.seq_start.numpy(), q_start, q_pos, pooled, topk)
    for s_, (p0, n) in enumerate(rows):
        s0 = int(b.seq_start[s_])
        Lmax = p0 + n
        k = b.k_cache[s0:s0 + Lmax].double().permute(1, 0, 2).repeat_interleave(2, 0)   # [Hq, Lmax, D]
        v = b.v_cache[s0:s0 + Lmax].double().permute(1, 0, 2).repeat_interleave(2, 0)
        qq = qf[q_start[s_]:q_start[s_ + 1]].double().permute(1, 0, 2)                   # [Hq, n, D]
        mask = torch.arange(Lmax)[None, :] <= (p0 + torch.arange(n))[:, None]           # [n, Lmax]
        o_ref = F.scaled_dot_product_attention(qq, k, v, attn_mask=mask).permute(1, 0, 2).numpy()
        np.testing.assert_allclose(out[q_start[s_]:q_start[s_ + 1]], o_ref, rtol=1e-10, atol=1e-12)
        logits = (qq @ k.transpose(-1, -2)) / math.sqrt(128)
        l_ref = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1).t().numpy()
        np.testing.assert_allclose(lse[q_start[s_]:q_start[s_ + 1]], l_ref, rtol=1e-12, atol=1e-12)
        for e in range(q_start[s_], q_start[s_ + 1]):
            L = p0 + (e - q_start[s_]) + 1
            assert (cnt[e] == oracle_mod.n_candidates(L)).all()
