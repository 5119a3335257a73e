"""Seeded synthetic inputs for NOSA sparse decode attention.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no pooling, scoring, selection or attention).  Both the
CUDA path's tests/benchmark and the CPU oracle's tests take their inputs from
here.

Layouts (shared with the C-ABI):
  * ``q``: bf16 ``[B, Hq, D]`` -- one decode query per sequence.
  * ``k_cache``/``v_cache``: bf16 ``[T, Hkv, D]``, token-major; sequence ``i``
    occupies rows ``[seq_start[i], seq_start[i] + capacity[i])`` of which the
    first ``seq_len[i]`` are filled.
  * ``seq_start``: int64 ``[B]``; ``seq_len``: int32 ``[B]``.

Workload shapes follow the NOSA-1B attention configuration (16 query heads,
2 KV heads, head_dim 128, bf16 -- "NOSA-1B 性能基准全解析" (wmrh.cn), §四 table)
and an 8B-class Llama shape (32 / 8 heads) that the pages do not spell out.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Sequence, Union

import torch


@dataclass
class DecodeBatch:
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    seq_start: torch.Tensor
    seq_len: torch.Tensor
    capacity: torch.Tensor
    num_q_heads: int
    num_kv_heads: int
    head_dim: int

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_len.max().item())

    def to(self, device) -> "DecodeBatch":
        return DecodeBatch(self.q.to(device), self.k_cache.to(device), self.v_cache.to(device),
                           self.seq_start.to(device), self.seq_len.to(device),
                           self.capacity.to(device), self.num_q_heads, self.num_kv_heads,
                           self.head_dim)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def ragged_lengths(batch: int, lo: int, hi: int, seed: int) -> list:
    """Sequence lengths drawn uniformly from [lo, hi] (inclusive), seeded."""
    g = _gen(seed, "cpu")
    return torch.randint(lo, hi + 1, (batch,), generator=g).tolist()


def _normal(shape, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _student_t(shape, nu: int, g, device) -> torch.Tensor:
    """Student-t with even ``nu`` degrees of freedom: Z / sqrt(chi2_nu / nu),
    chi2_nu = -2 * sum_{m < nu/2} log U_m."""
    assert nu % 2 == 0 and nu > 0
    z = _normal(shape, g, device)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(nu // 2):
        u = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
        chi2.add_(torch.log(u.clamp_min_(1e-30)), alpha=-2.0)
    return z / torch.sqrt(chi2 / nu)


def make_batch(seq_lens: Union[int, Sequence[int]], *, batch: Optional[int] = None,
               num_q_heads: int = 16, num_kv_heads: int = 2, head_dim: int = 128,
               seed: int = 0, key_dist: str = "normal", nu: int = 4, slack: int = 0,
               device="cpu") -> DecodeBatch:
    """q, K, V drawn i.i.d. (N(0,1), or Student-t(nu) keys), rounded to bf16.

    ``slack`` extra rows per sequence are reserved (and filled with random
    values) so that decode steps can append tokens in place."""
    if isinstance(seq_lens, int):
        assert batch is not None
        seq_lens = [seq_lens] * batch
    lens = [int(x) for x in seq_lens]
    B = len(lens)
    cap = [L + slack for L in lens]
    starts = [0]
    for c in cap[:-1]:
        starts.append(starts[-1] + c)
    T = sum(cap)
    g = _gen(seed, device)
    q = _normal((B, num_q_heads, head_dim), g, device).to(torch.bfloat16)
    if key_dist == "normal":
        k = _normal((T, num_kv_heads, head_dim), g, device)
    elif key_dist == "student_t":
        k = _student_t((T, num_kv_heads, head_dim), nu, g, device)
    else:
        raise ValueError(f"unknown key distribution {key_dist!r}")
    k = k.to(torch.bfloat16)
    v = _normal((T, num_kv_heads, head_dim), g, device).to(torch.bfloat16)
    return DecodeBatch(q, k, v,
                       torch.tensor(starts, dtype=torch.int64, device=device),
                       torch.tensor(lens, dtype=torch.int32, device=device),
                       torch.tensor(cap, dtype=torch.int32, device=device),
                       num_q_heads, num_kv_heads, head_dim)


def plant_blocks(b: DecodeBatch, *, planted_per_head: int = 8, ladder_step: float = 0.25,
                 margin: float = 2.0, seed: int = 0, block_size: int = 64,
                 local_blocks: int = 16, pool_kernel: int = 32) -> torch.Tensor:
    """Give every non-local block of every (sequence, KV head) a distinct,
    seeded amount of alignment with that group's queries (in place, CPU).

    For KV head g let u_g be the unit vector along the sum of the group's query
    vectors.  Non-local block c (c < number of blocks - local_blocks) gets
    lambda_c * u_g added to the keys of its middle ``pool_kernel`` tokens
    [c*bs + (bs - pool_kernel)/2, ... + pool_kernel), with
    lambda_c = ladder_step * rank_c, rank_c a seeded random permutation of the
    non-local blocks.  The ``planted_per_head`` blocks with the highest ranks
    get ``margin`` more.  Keys are then rounded back to bf16.

    Returns the planted block indices, int64 [B, Hkv, planted_per_head]
    (sorted ascending; -1 where a sequence has fewer candidates)."""
    assert b.k_cache.device.type == "cpu"
    g = _gen(seed, "cpu")
    G = b.num_q_heads // b.num_kv_heads
    off = (block_size - pool_kernel) // 2
    planted = torch.full((b.batch, b.num_kv_heads, planted_per_head), -1, dtype=torch.int64)
    k = b.k_cache.float()
    q = b.q.float()
    for i in range(b.batch):
        L = int(b.seq_len[i])
        nb = (L + block_size - 1) // block_size
        ncand = max(0, nb - local_blocks)
        if ncand == 0:
            continue
        base = int(b.seq_start[i])
        for h in range(b.num_kv_heads):
            u = q[i, h * G:(h + 1) * G].sum(0)
            u = u / u.norm()
            rank = torch.randperm(ncand, generator=g).to(torch.float32)
            lam = ladder_step * rank
            top = torch.argsort(rank, descending=True)[:planted_per_head]
            lam[top] += margin
            planted[i, h, :top.numel()] = torch.sort(top).values
            for c in range(ncand):
                r0 = base + c * block_size + off
                k[r0:r0 + pool_kernel, h] += lam[c] * u
    b.k_cache.copy_(k.to(torch.bfloat16))
    return planted


def random_queries(n: int, batch: int, num_q_heads: int, head_dim: int, seed: int,
                   device="cpu") -> torch.Tensor:
    """``n`` independent decode-query sets, bf16 [n, B, Hq, D]."""
    g = _gen(seed, device)
    return _normal((n, batch, num_q_heads, head_dim), g, device).to(torch.bfloat16)


def random_kv_rows(batch: int, num_kv_heads: int, head_dim: int, seed: int,
                   device="cpu"):
    """One new K row and V row per sequence, bf16 [B, Hkv, D] each."""
    g = _gen(seed, device)
    k = _normal((batch, num_kv_heads, head_dim), g, device).to(torch.bfloat16)
    v = _normal((batch, num_kv_heads, head_dim), g, device).to(torch.bfloat16)
    return k, v


def bf16_bits(t: torch.Tensor):
    """numpy uint16 view of a bf16 tensor's bit patterns (copies to host)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
