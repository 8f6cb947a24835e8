"""GPU: failure detection through bounded waits, made on purpose without any fault.

Every kernel bounds its mbarrier waits; past the limit a wait records FA_ERR_TIMEOUT in the
device status word and the kernel returns.  fa_selftest_wait_timeout runs that wait on a
barrier that nothing completes, with a 20 ms limit.  The kernel must end (no hang), the
status must read FA_ERR_TIMEOUT once and then be clear, and the context must stay usable."""

from __future__ import annotations

import pytest
import torch

import exact_attention_111_b200 as fa
from tests import parity as P

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_timeout():
    P.ensure_built()
    fa.fa_check_status()                               # start clean
    flag = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    fa.fa_selftest_wait_timeout(20000, flag, s)
    e1.record(s)
    torch.cuda.synchronize()
    assert flag.item() == 0                            # the wait gave up
    ms = e0.elapsed_time(e1)
    assert 20.0 <= ms < 2000.0, ms                     # at the limit, not forever
    with pytest.raises(fa.FAError) as e:
        fa.fa_check_status()
    assert e.value.code == fa.FA_ERR_TIMEOUT
    fa.fa_check_status()                               # the read cleared it


def test_context_usable_after_timeout():
    P.ensure_built()
    fa.fa_selftest_wait_timeout(1000)
    with pytest.raises(fa.FAError):
        fa.fa_check_status()
    inp = P.inputs(1, 2, 300, 64, seed=8100)
    o, lse, _ = P.gpu_forward(inp, True, None)         # checks the status word itself
    o_ref, lse_ref = P.oracle_forward(inp, True, None)
    P.check_forward(o, lse, o_ref, lse_ref, o16_dtype=torch.bfloat16, label="after timeout")
