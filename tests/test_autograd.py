"""The autograd wrapper SinkAttention: a loss through it gives the oracle's gradients for q,
k, v and the sink, plain and with dropout (the backward redraws the forward's keep bytes),
and the deterministic flag gives the same bits twice."""
import numpy as np
import pytest

import workloads as W
from oracle import ref
from _check import check_grad, check_out, to_np

pytestmark = pytest.mark.gpu


def _run(p, dropout=None, deterministic=False):
    import torch
    import softmax_attn_sink_b200 as sab
    from gpu_util import dev, tdtype
    td = tdtype(p)
    q, k, v = (dev(x, td).requires_grad_(True) for x in (p.q, p.k, p.v))
    sink = dev(p.sink).requires_grad_(True)
    cu_q, cu_k = dev(p.cu_seqlens_q), dev(p.cu_seqlens_k)
    out = sab.SinkAttention.apply(q, k, v, sink, cu_q, cu_k, max(p.max_seqlen_q, 1), max(p.max_seqlen_k, 1),
                                  p.softmax_scale, p.causal, p.window_left, p.window_right, dropout, deterministic)
    (out.float() * dev(p.dout).float()).sum().backward()
    torch.cuda.synchronize()
    return out, q.grad, k.grad, v.grad, sink.grad


@pytest.mark.parametrize("dropout", [None, (0.2, 77, 4)], ids=["plain", "dropout"])
def test_autograd_matches_oracle(dropout):
    p = W.random_problem(91, [200, 129], [230, 129], 4, 2, 128, 128, True, with_dout=True)
    out, dq, dk, dv, ds = _run(p, dropout)
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True, -1, -1)
    ro, _ = ref.fwd(p.q, p.k, p.v, *a, dropout=dropout)
    check_out(to_np(out), ro, "bf16")
    rdq, rdk, rdv, rds = ref.bwd(p.q, p.k, p.v, p.dout, *a, dropout=dropout)
    for name, g, r in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv), ("dsink", ds, rds)):
        check_grad(to_np(g), r, "bf16", name)


def test_autograd_deterministic_repeats():
    p = W.random_problem(92, [400, 300], [400, 300], 8, 2, 128, 128, True, with_dout=True)
    r1 = _run(p, deterministic=True)
    r2 = _run(p, deterministic=True)
    for x, y in zip(r1, r2):
        assert np.array_equal(to_np(x), to_np(y))
