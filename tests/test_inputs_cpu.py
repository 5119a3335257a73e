"""The seeded input recipe: layouts, determinism and value distributions of
the synthetic workloads (N(0,1) q / K / V, Student-t(4) keys for the
8B-class shape, ragged lengths uniform on [16K, 32K])."""
import numpy as np
import pytest
import torch
from scipy import stats

from long_context_decode_nosa_b200 import inputs


def test_layout_and_capacity():
    b = inputs.make_batch([5, 70, 1], num_q_heads=4, num_kv_heads=2, seed=3, slack=10)
    assert b.q.shape == (3, 4, 128) and b.q.dtype == torch.bfloat16
    assert b.k_cache.shape == (15 + 80 + 11, 2, 128) and b.v_cache.shape == b.k_cache.shape
    assert b.seq_start.tolist() == [0, 15, 95] and b.seq_start.dtype == torch.int64
    assert b.seq_len.tolist() == [5, 70, 1] and b.seq_len.dtype == torch.int32
    assert b.capacity.tolist() == [15, 80, 11]
    assert b.batch == 3 and b.max_seq_len == 70


def test_seeded_and_deterministic():
    a = inputs.make_batch(300, batch=2, seed=11)
    b = inputs.make_batch(300, batch=2, seed=11)
    c = inputs.make_batch(300, batch=2, seed=12)
    for x, y in ((a.q, b.q), (a.k_cache, b.k_cache), (a.v_cache, b.v_cache)):
        assert torch.equal(x, y)
    assert not torch.equal(a.k_cache, c.k_cache)
    assert inputs.ragged_lengths(32, 16384, 32768, seed=3) == inputs.ragged_lengths(32, 16384, 32768, seed=3)


def test_normal_values():
    b = inputs.make_batch(4096, batch=4, seed=5)
    for t in (b.q, b.k_cache, b.v_cache):
        x = t.float().flatten().numpy()
        tol = 5.0 / np.sqrt(x.size)  # five standard errors
        assert abs(x.mean()) < tol and abs(x.std() - 1.0) < tol
        # bf16 values: 8 significant bits
        assert torch.equal(t.float().to(torch.bfloat16).float(), t.float())


def test_student_t_keys():
    """Keys with key_dist="student_t" follow Student-t with 4 degrees of
    freedom (its variance has no finite estimate error, so quantiles are
    compared); q and V stay N(0,1)."""
    b = inputs.make_batch(16384, batch=2, num_q_heads=32, num_kv_heads=8, seed=4, key_dist="student_t")
    k = b.k_cache.float().flatten().numpy()
    for p in (0.75, 0.9, 0.99, 0.999):
        want = stats.t.ppf(p, df=4)
        assert abs(np.quantile(k, p) - want) < 0.02 * want + 0.01, p
        assert abs(np.quantile(k, 1 - p) + want) < 0.02 * want + 0.01, p
    v = b.v_cache.float().flatten().numpy()
    assert abs(np.quantile(v, 0.99) - stats.norm.ppf(0.99)) < 0.02


def test_ragged_lengths_uniform_inclusive():
    lens = np.array(inputs.ragged_lengths(20000, 16384, 32768, seed=7))
    assert lens.min() >= 16384 and lens.max() <= 32768
    assert abs(lens.mean() - (16384 + 32768) / 2) < 150
    assert stats.kstest((lens - 16384) / (32768 - 16384 + 1), "uniform").pvalue > 1e-3


def test_unknown_key_distribution_rejected():
    with pytest.raises(ValueError):
        inputs.make_batch(10, batch=1, key_dist="cauchy")
