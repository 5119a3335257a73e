"""The scratch-free decode step (B200).

nosa_decode_step_device_noalloc serves callers that cannot allocate device
memory -- e.g. an engine plugin whose host owns the whole device pool and
offers no workspace, or a serving loop that may not call cudaMalloc once the
KV cache has taken the free memory.  It runs the fused step with the library's
own fixed device scratch instead of a workspace.  These tests call it through
the C ABI twice in a row and check each result against the workspace entry
point, within the parity tolerances used everywhere else.  This file is
collected last so that a stop-at-first-failure run has run every other test.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from helpers import LSE_ATOL, assert_out_close
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


def test_noalloc_matches_workspace_entry_point_on_two_calls(nosa):
    lens = [16384, 9000, 5000, 1100, 3000, 12000, 700, 16384]
    b = inputs.make_batch(lens, num_q_heads=16, num_kv_heads=2, seed=77, device=DEV)
    p = nosa.params(16, 2, topk=64)
    ref = nosa.DecodeState(p, b.batch, b.max_seq_len)
    ref.rebuild_pooled(b.k_cache, b.seq_start, b.seq_len)
    ref.step(b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len, fused=True, with_lse=True)
    torch.cuda.synchronize()
    out_ref = ref.out.float().cpu().numpy()
    lse_ref = ref.lse.cpu().numpy()
    sel_ref, cnt_ref = ref.sel_idx.cpu(), ref.sel_cnt.cpu()

    pooled = ref.pooled.clone()
    for call in range(2):
        sel = torch.full_like(ref.sel_idx, -7)
        cnt = torch.full_like(ref.sel_cnt, -7)
        out = torch.full_like(ref.out, float("nan"))
        lse = torch.full_like(ref.lse, float("nan"))
        nosa.nosa_decode_step_device_noalloc(p, b.q, b.k_cache, b.v_cache, b.seq_start, b.seq_len,
                                             b.max_seq_len, pooled, sel, cnt, out, lse=lse)
        torch.cuda.synchronize()
        assert_out_close(out.float().cpu().numpy(), out_ref)
        np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, atol=LSE_ATOL, rtol=0)
        assert torch.equal(cnt.cpu(), cnt_ref) and torch.equal(sel.cpu(), sel_ref), call
    assert torch.equal(pooled, ref.pooled)


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
