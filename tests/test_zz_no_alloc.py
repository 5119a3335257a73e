"""The scratch-free decode step (B200).

nosa_decode_step_device_noalloc serves callers that cannot allocate device
memory -- e.g. an engine plugin whose host owns the whole device pool and
offers no workspace, or a serving loop that may not call cudaMalloc once the
KV cache has taken the free memory.  It runs the fused step with the library's
own fixed device scratch instead of a workspace.  These tests call it through
the C ABI twice in a row and check each result against the workspace entry
point: both launch the same kernel with the same cluster size, so outputs,
log-sum-exps and selections must be identical bit for bit.  One case keeps
its block scores in the built-in array (sequences beyond 2048 candidates), so
the second call also reads a region the first one left behind.  This file is
collected last so that a stop-at-first-failure run has run every other test.
"""
from __future__ import annotations

import pytest
import torch

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


def _two_calls_match_workspace_call(nosa, lens, seed):
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=seed, device=DEV)
    p = nosa.params(16, 2, topk=64)
    ref = nosa.DecodeState(p, b.batch, b.max_seq_len)
    ref.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
    ref.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, fused=True, with_lse=True)
    torch.cuda.synchronize()
    pooled = ref.pooled.clone()
    for call in range(2):
        sel = torch.full_like(ref.sel_idx, -7)
        cnt = torch.full_like(ref.sel_cnt, -7)
        out = torch.full_like(ref.out, float("nan"))
        lse = torch.full_like(ref.lse, float("nan"))
        nosa.nosa_decode_step_device_noalloc(p, b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len,
                                             b.max_seq_len, pooled, sel, cnt, out, lse=lse)
        torch.cuda.synchronize()
        assert torch.equal(cnt, ref.sel_cnt) and torch.equal(sel, ref.sel_idx), call
        assert torch.equal(out, ref.out) and torch.equal(lse, ref.lse), call
    assert torch.equal(pooled, ref.pooled)


def test_noalloc_matches_workspace_entry_point_on_two_calls(nosa):
    _two_calls_match_workspace_call(nosa, [16384, 9000, 5000, 1100, 3000, 12000, 700, 16384], 77)


def test_noalloc_spilled_block_scores_on_two_calls(nosa):
    # 150000 tokens: 2328 candidates, beyond the 2048 that shared memory
    # holds, so the block scores of both sequences live in the built-in array.
    p = nosa.params(16, 2, topk=64)
    lens = [150000, 140000]
    assert nosa.workspace_size(p, 2, max(lens)) > nosa.workspace_size(p, 2, 16384)
    _two_calls_match_workspace_call(nosa, lens, 78)


def test_noalloc_rejects_a_batch_beyond_its_scratch(nosa):
    # 64 sequences of up to 2^20 tokens keep their block scores in scratch
    # (16368 candidates each, beyond what shared memory holds): more than the
    # built-in 8 MiB.  The call is refused before anything is launched.
    p = nosa.params(16, 2, topk=64)
    assert nosa.workspace_size(p, 64, 1 << 20) > 8 << 20
    one = torch.zeros(1, dtype=torch.bfloat16, device=DEV)
    i64 = torch.zeros(64, dtype=torch.int64, device=DEV)
    i32 = torch.ones(64, dtype=torch.int32, device=DEV)
    with pytest.raises(nosa.NosaError) as err:
        nosa.nosa_decode_step_device_noalloc(
            p, one.expand(64, 16, 128).contiguous(), one.expand(8, 2, 128).contiguous(),
            one.expand(8, 2, 128).contiguous(), i64, i32, 1 << 20,
            torch.zeros(64, 2, 1, 128, device=DEV), torch.zeros(64, 2, 64, dtype=torch.int32, device=DEV),
            torch.zeros(64, 2, dtype=torch.int32, device=DEV),
            torch.zeros(64, 16, 128, dtype=torch.bfloat16, device=DEV))
    assert err.value.code == nosa.NOSA_ERR_WORKSPACE
    assert "8388608" in str(err.value)
