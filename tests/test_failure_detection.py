"""Failure detection without a GPU fault: the tensor-core kernels give every on-chip wait a
time limit and report a timeout through a per-device status word instead of hanging.  The
diagnostics entry point makes one such wait run out on purpose (a barrier nothing
completes); the host reads the timeout, and the same context then still computes correct
results."""
import pytest

import workloads as W
from oracle import ref
from _check import check_lse, check_out, to_np

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import torch
    import softmax_attn_sink_b200 as sab
    st, bits = sab.device_status()
    assert st == 0 and bits == 0          # clean before
    sab.selftest_wait_timeout()
    st, bits = sab.device_status()
    assert st == 5 and bits & 1           # ATTN_SINK_ERR_TIMEOUT, timeout bit
    st, bits = sab.device_status()
    assert st == 0 and bits == 0          # reading clears it
    # the context is still usable: a tensor-core forward still matches the oracle
    from gpu_util import run_fwd
    p = W.random_problem(77, [200, 129], [200, 129], 4, 2, 128, 128, True)
    out, lse = run_fwd(p)
    ro, rl = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True)
    check_out(to_np(out), ro, "bf16")
    check_lse(to_np(lse), rl, "bf16")
    assert sab.device_status()[0] == 0


@pytest.mark.parametrize("case,expect", [
    (dict(), 0),
    (dict(cu_k=[0, 5, 3, 10]), 6),          # decreasing
    (dict(cu_k=[1, 5, 7, 10]), 6),          # does not start at 0
    (dict(cu_k=[0, 5, 7, 9]), 6),           # does not end at total_k
    (dict(cu_q=[0, 4, 4, 8]), 0),           # an empty sequence is fine
    (dict(max_q=3), 6),                     # a sequence longer than max_seqlen_q
])
def test_check_seqlens_reports_broken_contract(case, expect):
    """cu_seqlens live on the device, so their contract is checked there: a violation sets
    the status word, which reads back as ATTN_SINK_ERR_BAD_INDEX (6)."""
    import torch
    import softmax_attn_sink_b200 as sab
    cu_q = torch.tensor(case.get("cu_q", [0, 4, 6, 8]), dtype=torch.int32, device="cuda")
    cu_k = torch.tensor(case.get("cu_k", [0, 5, 7, 10]), dtype=torch.int32, device="cuda")
    sab.device_status()
    st, bits = sab.check_seqlens(cu_q, cu_k, 8, 10, case.get("max_q", 4), 5)
    assert st == expect, (st, bits)
