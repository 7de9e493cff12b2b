"""Failure detection without a GPU fault: a kernel's bounded wait that cannot
complete gives up, the host reads B200ATTN_ERR_TIMEOUT through b200attn_check,
and the context keeps working afterwards."""
import pytest
import torch

import oracle
import workloads
import bf16_causal_prefill_fwd_b200 as b2
from helpers import BF16_TOL, f32

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert b2.check() == 0
    b2.selftest_wait_timeout(limit_us=20000)
    assert b2.check() == -4          # reported once ...
    assert b2.check() == 0           # ... and cleared
    q, k, v = workloads.draw(workloads.gaussian(1, 2, 1, 300, 128, 128, seed=3))
    o = b2.attn_fwd(q.cuda(), k.cuda(), v.cuda())
    assert b2.check() == 0
    ref, _ = oracle.attention(f32(q), f32(k), f32(v))
    assert oracle.rel_rms(f32(o), ref) <= BF16_TOL


def test_selftest_rejects_bad_limit():
    with pytest.raises(b2.B200AttnError):
        b2.selftest_wait_timeout(limit_us=0)
